"""A round driver over the C ABI: owns the per-batch device buffers and issues, per round,
select -> k x (sparse draft attention, [draft logits], draft sampling) -> dense verify ->
[target logits] -> speculative sampling -> commit, all on one stream and all in libs3r.so.

The logits between attention and sampling belong to the rest of the model; callers pass
them in (synthetic workloads) or fill them from the attention outputs through the
optional callbacks (a projection, as in the budget sweep).
"""
from __future__ import annotations

import torch

from . import _lib as L


def budget_count(length: int, budget_bp: int, window: int) -> int:
    """Size n of the sparse set at committed length `length` (host-side mirror for sizing)."""
    n = -(-(length * budget_bp) // 10000)
    w = min(window, length)
    return min(max(n, w), length)


class RoundBuffers:
    """Device buffers of one batch: selection, attention outputs, tokens and statistics.

    The buffers whose layout depends on the draft length hold k_max drafts; set_k(k) makes
    the attributes contiguous views laid out for k (the layouts the library's calls use), so
    the draft length can change between rounds."""

    def __init__(self, num_requests, num_q_heads, num_kv_heads, head_dim, cap, k_max, vocab,
                 sel_stride, device="cuda"):
        self.dims = (num_requests, num_q_heads, num_kv_heads, head_dim, cap)
        G = num_q_heads // num_kv_heads
        f32, bf, i32 = torch.float32, torch.bfloat16, torch.int32
        T = k_max + 1
        self.k_max = k_max
        self._scores = torch.empty(num_requests * num_kv_heads * G * T * cap, dtype=f32, device=device)
        self._lse = torch.empty(num_requests * T * num_q_heads, dtype=f32, device=device)
        self._verify_out = torch.empty(num_requests * T * num_q_heads * head_dim, dtype=bf, device=device)
        self._draft_tokens = torch.zeros(num_requests * k_max, dtype=i32, device=device)
        self._out_tokens = torch.full((num_requests * T,), -1, dtype=i32, device=device)
        # decision margins the samplers report (draft draws; accept tests and the final draw)
        self._draft_margins = torch.zeros(num_requests * k_max, dtype=f32, device=device)
        self._spec_margins = torch.zeros(num_requests * T, dtype=f32, device=device)
        # the draft rows' normalisers (s3r_row_norm), written by the draft sampler and read by
        # the speculative sampler instead of streaming the q rows again
        self._q_norm = torch.zeros(num_requests * k_max * 2, dtype=torch.float64, device=device)
        self.prefill_lse = torch.empty((num_requests, 1, num_q_heads), dtype=f32, device=device)
        self.sel_idx = torch.zeros((num_requests, num_kv_heads, sel_stride), dtype=i32, device=device)
        self.sel_count = torch.zeros((num_requests, num_kv_heads), dtype=i32, device=device)
        self.steps = [torch.full((num_requests,), i, dtype=i32, device=device) for i in range(k_max)]
        self.draft_out = torch.empty((num_requests, num_q_heads, head_dim), dtype=bf, device=device)
        self.draft_lse = torch.empty((num_requests, num_q_heads), dtype=f32, device=device)
        self.n_out = torch.zeros((num_requests,), dtype=i32, device=device)
        # [0] tokens, [1] request-rounds, [2 + j] accepted / [2 + MAX_K + j] decided at position j
        self.stats = torch.zeros((2 + 2 * L.MAX_K,), dtype=torch.int64, device=device)
        self.set_k(k_max)

    def set_k(self, k: int):
        NR, Hq, Hkv, d, cap = self.dims
        G, T = Hq // Hkv, k + 1
        self.scores = self._scores[: NR * Hkv * G * T * cap].view(NR, Hkv, G * T, cap)
        self.lse = self._lse[: NR * T * Hq].view(NR, T, Hq)
        self.verify_out = self._verify_out[: NR * T * Hq * d].view(NR, T, Hq, d)
        self.draft_tokens = self._draft_tokens[: NR * k].view(NR, k)
        self.out_tokens = self._out_tokens[: NR * T].view(NR, T)
        self.draft_margins = self._draft_margins[: NR * k].view(NR, k)
        self.spec_margins = self._spec_margins[: NR * T].view(NR, T)
        self.q_norm = self._q_norm[: NR * k * 2].view(NR, k, 2)


class S3REngine:
    """S3R rounds for a batch of requests over one paged KV cache on one GPU."""

    def __init__(self, k_pool, v_pool, page_table, seq_lens, num_q_heads, *, k, budget_bp,
                 window, vocab, seed, sel_stride=None, greedy=False, page_select=False, k_max=None,
                 overlap_scores=True):
        k_max = k if k_max is None else k_max
        if not (1 <= k <= k_max <= L.MAX_K):
            raise ValueError("need 1 <= k <= k_max <= 8")
        self.k, self.budget_bp, self.window, self.vocab, self.seed = k, budget_bp, window, vocab, seed
        self.greedy = greedy   # temperature 0: argmax drafts, greedy verification
        self.page_select = page_select   # whole 16-position pages instead of positions
        self.k_pool, self.v_pool = k_pool, v_pool
        self.page_table = page_table
        self.seq_lens = seq_lens
        self.cache = L.make_cache(k_pool, v_pool, num_q_heads)
        self.num_requests, self.max_pages = page_table.shape
        self.cap = self.max_pages * L.PAGE_SIZE
        # a page-granular set holds up to 15 positions more than the token budget
        self.sel_stride = sel_stride or (budget_count(self.cap, budget_bp, window)
                                         + (L.PAGE_SIZE - 1 if page_select else 0))
        self.buf = RoundBuffers(self.num_requests, num_q_heads, self.cache.num_kv_heads,
                                self.cache.head_dim, self.cap, k_max, vocab, self.sel_stride,
                                k_pool.device)
        self.buf.set_k(k)
        nbytes = L.s3r_workspace_size(self.cache, self.num_requests, self.max_pages, k_max, vocab,
                                      self.sel_stride)
        self.ws = L.new_workspace(nbytes, k_pool.device)
        self.batch = L.make_batch(seq_lens, page_table)
        # The next selection's position scores (s3r_position_scores) are computed on a second
        # stream while speculative sampling and the commit run on this one; they read the
        # lengths from a snapshot taken before the fork, so the commit never races them.
        self.overlap_scores = overlap_scores
        self._scores_ready = False
        if overlap_scores:
            self.pos_scores = torch.empty((self.num_requests, self.cache.num_kv_heads, self.cap),
                                          dtype=torch.float32, device=k_pool.device)
            self._len_snap = torch.empty_like(seq_lens)
            self._snap_batch = L.make_batch(self._len_snap, page_table)
            self._score_stream = torch.cuda.Stream(k_pool.device)
        self.k_prev = None
        self._verify_launches = 2

    def set_k(self, k: int):
        """Draft length of the next rounds (1 <= k <= k_max). The selection of the next round
        still reads the last verify's scores with that verify's length (k_prev)."""
        if not (1 <= k <= self.buf.k_max):
            raise ValueError("k outside 1..k_max")
        self.k = k
        self.buf.set_k(k)

    @property
    def launches_per_round(self) -> int:
        # select (scores + select), k x (draft, sample), verify (attention launches + the chunk
        # merge, as counted at the last verify), spec (2 / 1 greedy), commit
        return 2 + 2 * self.k + self._verify_launches + (1 if self.greedy else 2) + 1

    def prefill(self, q_x, k_x, v_x):
        """One-row dense pass of each request's pending token at position L (the last step of
        a prefill): writes its K/V and the scores the first selection reads.
        q_x [NR][1][H_q][d], k_x / v_x [NR][1][H_kv][d]."""
        b = self.buf
        out = torch.empty_like(q_x)
        L.s3r_verify_attn(self.cache, self.batch, 0, q_x, k_x, v_x, out, b.prefill_lse, b.scores,
                          self.ws)
        self.k_prev = 0
        return out

    def select(self):
        b = self.buf
        if self._scores_ready:   # the scores computed beside the last round's sampling
            fn = L.s3r_select_pages_from_scores if self.page_select else L.s3r_select_from_scores
            fn(self.cache, self.batch, self.pos_scores, self.budget_bp, self.window, b.sel_idx,
               b.sel_count, self.ws)
            return
        lse = b.prefill_lse if self.k_prev == 0 else b.lse
        fn = L.s3r_select_kv_pages if self.page_select else L.s3r_select_kv
        fn(self.cache, self.batch, b.scores, lse, self.k_prev, self.budget_bp, self.window,
           b.sel_idx, b.sel_count, self.ws)

    def draft_attn(self, i, q_block, k_block, v_block):
        b = self.buf
        L.s3r_sparse_draft_attn(self.cache, self.batch, b.steps[i], q_block[:, i], k_block[:, i],
                                v_block[:, i], b.sel_idx, b.sel_count, b.draft_out, b.draft_lse,
                                self.ws)

    def draft_sample(self, i, q_logits):
        if self.greedy:
            L.s3r_draft_argmax(self.batch, self.buf.steps[i], self.k, q_logits, self.vocab,
                               self.buf.draft_tokens, self.ws)
            return
        L.s3r_draft_sample(self.batch, self.buf.steps[i], self.k, q_logits, self.vocab, self.seed,
                           self.buf.draft_tokens, self.ws, margins=self.buf.draft_margins,
                           q_norm=self.buf.q_norm)

    def draft_step(self, i, q_block, k_block, v_block, q_logits, draft_logits_fn=None):
        self.draft_attn(i, q_block, k_block, v_block)
        if draft_logits_fn is not None:
            draft_logits_fn(i, self.buf.draft_out, q_logits)
        self.draft_sample(i, q_logits)

    def verify(self, q_block, k_block, v_block):
        b = self.buf
        before = L.s3r_launch_count()
        L.s3r_verify_attn(self.cache, self.batch, self.k, q_block, k_block, v_block, b.verify_out,
                          b.lse, b.scores, self.ws)
        self._verify_launches = L.s3r_launch_count() - before
        self.k_prev = self.k
        self._scores_ready = False

    def fork_scores(self, batch, snap_batch, k):
        """The position scores of the verify just run, for the batch's requests, on the second
        stream (lengths from a snapshot of seq_lens); join_scores() rejoins it."""
        main = torch.cuda.current_stream()
        self._len_snap.copy_(self.seq_lens, non_blocking=True)
        self._score_stream.wait_stream(main)
        with torch.cuda.stream(self._score_stream):
            L.s3r_position_scores(self.cache, snap_batch, self.buf.scores, self.buf.lse, k,
                                  self.pos_scores, self.ws)

    def join_scores(self):
        torch.cuda.current_stream().wait_stream(self._score_stream)

    def sample_and_commit(self, p_logits, q_logits):
        b = self.buf
        if self.overlap_scores:
            self.fork_scores(self.batch, self._snap_batch, self.k)
        if self.greedy:
            L.s3r_greedy_verify(self.batch, self.k, p_logits, b.draft_tokens, self.vocab,
                                b.out_tokens, b.n_out, self.ws)
        else:
            L.s3r_spec_sample(self.batch, self.k, p_logits, q_logits, b.draft_tokens, self.vocab,
                              self.seed, b.out_tokens, b.n_out, self.ws, margins=b.spec_margins,
                              q_norm=b.q_norm)
        L.s3r_commit(self.batch, self.k, b.n_out, self.seq_lens, b.stats)
        if self.overlap_scores:
            self.join_scores()
            self._scores_ready = True

    def round(self, q_block, k_block, v_block, p_logits, q_logits, draft_logits_fn=None,
              target_logits_fn=None):
        """One draft+verify round for every request.

        q_block [NR][k+1][H_q][d], k_block / v_block [NR][k+1][H_kv][d]: projections of the
        tokens at positions L..L+k; p_logits [NR][k+1][V], q_logits [NR][k][V] (filled by the
        callbacks when given)."""
        if self.k_prev is None:
            raise RuntimeError("call prefill() before the first round")
        self.select()
        for i in range(self.k):
            self.draft_step(i, q_block, k_block, v_block, q_logits, draft_logits_fn)
        self.verify(q_block, k_block, v_block)
        if target_logits_fn is not None:
            target_logits_fn(self.buf.verify_out, p_logits)
        self.sample_and_commit(p_logits, q_logits)

    def check_errors(self) -> int:
        """Synchronise and return (and clear) the device error bitmask."""
        return L.s3r_get_error(self.ws)

    def capture(self, step):
        """Record `step()` (library calls on fixed device buffers) into a CUDA graph once;
        replaying it issues the same launches with no host work per launch. `step` runs once
        eagerly on a side stream first, so one-time host set-up (kernel attributes) is done
        before capture. Returns (graph, launches recorded per replay)."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        before = L.s3r_launch_count()
        with torch.cuda.graph(g):
            step()
        return g, L.s3r_launch_count() - before


class MixedPhaseDriver:
    """Requests at different points of their rounds, advanced one phase per iteration with
    launches over request subsets (req_ids): phase i < k is draft step i, phase k is the
    verify, speculative sampling and commit, followed at once by the selection of the
    request's next round. One iteration issues one draft-attention and one draft-sampling
    launch for every drafting request (each reads its own step from the step array), one
    verify, one speculative-sampling pass, one commit and one selection for the verifying
    requests.

    Which request is in which phase is host bookkeeping (a numpy array); the kernels see only
    the request-id lists and the per-request step array.
    """

    def __init__(self, engine: S3REngine, phases):
        import numpy as np
        self.e = engine
        self.phases = np.asarray(phases, dtype=np.int64).copy()
        if self.phases.shape != (engine.num_requests,) or self.phases.min() < 0 or \
                self.phases.max() > engine.k:
            raise ValueError("one phase in 0..k per request")
        dev = engine.k_pool.device
        self.step = torch.zeros((engine.num_requests,), dtype=torch.int32, device=dev)
        self._dev = dev

    def _batch(self, ids, snap=False):
        t = torch.as_tensor(ids, dtype=torch.int32, device=self._dev)
        lens = self.e._len_snap if snap else self.e.seq_lens
        return L.make_batch(lens, self.e.page_table, req_ids=t)

    def _reselect(self, vb, v_snap, k, commit):
        """Verify done for the batch vb: position scores (beside the sampling and commit when
        the engine overlaps them), `commit()`, then the new sparse sets."""
        e, b = self.e, self.e.buf
        if e.overlap_scores:
            e.fork_scores(vb, v_snap, k)
        commit()
        if e.overlap_scores:
            e.join_scores()
            sel = L.s3r_select_pages_from_scores if e.page_select else L.s3r_select_from_scores
            sel(e.cache, vb, e.pos_scores, e.budget_bp, e.window, b.sel_idx, b.sel_count, e.ws)
        else:
            sel = L.s3r_select_kv_pages if e.page_select else L.s3r_select_kv
            sel(e.cache, vb, b.scores, b.lse, k, e.budget_bp, e.window, b.sel_idx, b.sel_count, e.ws)

    def start(self, q_block, k_block, v_block, q_logits):
        """After prefill: every request selects its first sparse set from the prefill scores,
        then drafts the steps before its phase (a request at phase p has drafted 0..p-1)."""
        import numpy as np
        e = self.e
        e.select()
        for i in range(e.k):
            ids = np.nonzero(self.phases > i)[0]
            if ids.size:
                self._draft(ids, np.full(ids.size, i), q_block, k_block, v_block, q_logits)

    def _draft(self, ids, steps, q_block, k_block, v_block, q_logits):
        import numpy as np
        e, b = self.e, self.e.buf
        st = np.zeros(e.num_requests, dtype=np.int32)
        st[ids] = steps
        self.step.copy_(torch.as_tensor(st), non_blocking=False)
        rows = torch.as_tensor(st, dtype=torch.long, device=self._dev)
        ar = torch.arange(e.num_requests, device=self._dev)
        # the current token of each request (its own step) -- model output in a real system
        qc = q_block[ar, rows].contiguous()
        kc = k_block[ar, rows].contiguous()
        vc = v_block[ar, rows].contiguous()
        batch = self._batch(ids)
        L.s3r_sparse_draft_attn(e.cache, batch, self.step, qc, kc, vc, b.sel_idx, b.sel_count,
                                b.draft_out, b.draft_lse, e.ws)
        if e.greedy:
            L.s3r_draft_argmax(batch, self.step, e.k, q_logits, e.vocab, b.draft_tokens, e.ws)
        else:
            L.s3r_draft_sample(batch, self.step, e.k, q_logits, e.vocab, e.seed, b.draft_tokens,
                               e.ws, margins=b.draft_margins, q_norm=b.q_norm)

    def cycle(self, q_block, k_block, v_block, p_logits, q_logits):
        """The k+1 iterations of one cycle from the current phases, as callables that issue
        only library launches on fixed device buffers (so each can be captured in a CUDA
        graph and replayed): iteration c drafts every request at phase (phase0 + c) % (k+1)
        < k and verifies, samples, commits and reselects the others. The request lists, the
        step arrays and each drafting request's current q/k/v rows are gathered here, once,
        on the device. Calling them in order 0..k advances every request by one round and
        returns the phases to where they were. Each callable takes an optional dict of
        CUDA events ("d0", "dm", "d1", "v0", "v1", "c1", "s1") recorded between its calls."""
        import numpy as np
        e, b = self.e, self.e.buf
        k, NR, dev = e.k, e.num_requests, self._dev
        ar = torch.arange(NR, device=dev)
        its = []
        for c in range(k + 1):
            ph = (self.phases + c) % (k + 1)
            d_ids = np.nonzero(ph < k)[0]
            v_ids = np.nonzero(ph == k)[0]
            st = np.zeros(NR, dtype=np.int32)
            st[d_ids] = ph[d_ids]
            st_d = torch.as_tensor(st, device=dev)
            rows = st_d.long()
            it = dict(n_draft=int(d_ids.size), n_verify=int(v_ids.size), d_ids=d_ids, v_ids=v_ids,
                      steps=st, step=st_d, qc=q_block[ar, rows].contiguous(),
                      kc=k_block[ar, rows].contiguous(), vc=v_block[ar, rows].contiguous(),
                      d_batch=self._batch(d_ids) if d_ids.size else None,
                      v_batch=self._batch(v_ids) if v_ids.size else None,
                      v_snap=self._batch(v_ids, snap=True) if v_ids.size and e.overlap_scores else None)
            its.append(it)

        def make(it):
            def run(ev=None):
                rec = (lambda n: ev[n].record()) if ev is not None else (lambda n: None)
                rec("d0")
                if it["n_draft"]:
                    L.s3r_sparse_draft_attn(e.cache, it["d_batch"], it["step"], it["qc"], it["kc"], it["vc"],
                                            b.sel_idx, b.sel_count, b.draft_out, b.draft_lse, e.ws)
                rec("dm")
                if it["n_draft"]:
                    if e.greedy:
                        L.s3r_draft_argmax(it["d_batch"], it["step"], k, q_logits, e.vocab, b.draft_tokens, e.ws)
                    else:
                        L.s3r_draft_sample(it["d_batch"], it["step"], k, q_logits, e.vocab, e.seed,
                                           b.draft_tokens, e.ws, margins=b.draft_margins, q_norm=b.q_norm)
                rec("d1")
                rec("v0")
                if it["n_verify"]:
                    vb = it["v_batch"]
                    L.s3r_verify_attn(e.cache, vb, k, q_block, k_block, v_block, b.verify_out, b.lse,
                                      b.scores, e.ws)
                    rec("v1")

                    def commit():
                        if e.greedy:
                            L.s3r_greedy_verify(vb, k, p_logits, b.draft_tokens, e.vocab, b.out_tokens,
                                                b.n_out, e.ws)
                        else:
                            L.s3r_spec_sample(vb, k, p_logits, q_logits, b.draft_tokens, e.vocab, e.seed,
                                              b.out_tokens, b.n_out, e.ws, margins=b.spec_margins,
                                              q_norm=b.q_norm)
                        L.s3r_commit(vb, k, b.n_out, e.seq_lens, b.stats)
                        rec("c1")
                    self._reselect(vb, it["v_snap"], k, commit)
                else:
                    rec("v1")
                    rec("c1")
                rec("s1")
            run.info = it
            return run

        return [make(it) for it in its]

    def iterate(self, q_block, k_block, v_block, p_logits, q_logits):
        """Advance every request by one phase; returns the ids that completed a round."""
        import numpy as np
        e, b = self.e, self.e.buf
        d_ids = np.nonzero(self.phases < e.k)[0]
        v_ids = np.nonzero(self.phases == e.k)[0]
        if d_ids.size:
            self._draft(d_ids, self.phases[d_ids], q_block, k_block, v_block, q_logits)
        if v_ids.size:
            batch = self._batch(v_ids)
            L.s3r_verify_attn(e.cache, batch, e.k, q_block, k_block, v_block, b.verify_out, b.lse,
                              b.scores, e.ws)

            def commit():
                if e.greedy:
                    L.s3r_greedy_verify(batch, e.k, p_logits, b.draft_tokens, e.vocab, b.out_tokens,
                                        b.n_out, e.ws)
                else:
                    L.s3r_spec_sample(batch, e.k, p_logits, q_logits, b.draft_tokens, e.vocab,
                                      e.seed, b.out_tokens, b.n_out, e.ws, margins=b.spec_margins,
                                      q_norm=b.q_norm)
                L.s3r_commit(batch, e.k, b.n_out, e.seq_lens, b.stats)
            self._reselect(batch, self._batch(v_ids, snap=True) if e.overlap_scores else None, e.k,
                           commit)
        self.phases = (self.phases + 1) % (e.k + 1)
        return v_ids


class AdaptiveHorizon:
    """Draft length from the measured acceptance by position: every call of step() reads the
    engine's counters (one device-to-host copy) and s3r_horizon_step decays the kept counts,
    adds the new ones, takes the prior and picks the k with the most expected tokens per unit
    round cost: c_draft per draft step plus c_verify for the rest of the round, or, with
    round_costs, the measured cost of a round at each length 1..k_max
    (s3r_horizon_step_costs). Positions not drafted for a while decay toward the prior, so
    longer horizons are tried again when it is good; with prior_alpha="pooled" the prior is
    the acceptance pooled over all positions so far (the plain expectation for a position
    without evidence of its own). With stale_counts the counters are copied asynchronously
    and each decision reads the copy started at the previous one, so the host never waits
    for the device (the decisions lag the counts by one interval)."""

    def __init__(self, engine: S3REngine, c_draft: float = 0.0, c_verify: float = 0.0, *, decay: float = 0.8,
                 prior_alpha="pooled", prior_weight: float = 4.0, k_max: int | None = None,
                 round_costs=None, stale_counts: bool = False):
        import numpy as np
        self.e = engine
        self.c_draft, self.c_verify = c_draft, c_verify
        # round_costs: the cost of a round at each length 1..k_max, used instead of the line
        # k * c_draft + c_verify when given
        self.round_costs = None if round_costs is None else [float(c) for c in round_costs]
        if self.round_costs is None and not (c_draft > 0 and c_verify > 0):
            raise ValueError("give c_draft and c_verify (> 0) or round_costs")
        self.decay, self.prior_alpha, self.prior_weight = decay, prior_alpha, prior_weight
        self.k_max = k_max or engine.buf.k_max
        self.acc = np.zeros(L.MAX_K, dtype=np.float64)
        self.dec = np.zeros(L.MAX_K, dtype=np.float64)
        self.last = engine.buf.stats.cpu().numpy().astype(np.int64)
        self.last_prior = None
        self.history = []
        # stale_counts: each decision reads the counters copied (asynchronously, into pinned
        # memory) at the previous decision, so the host never waits for the device; the
        # decisions then lag the counts by one interval
        self.stale = stale_counts
        self._host = None
        self._copied = None

    def _counters(self):
        import numpy as np
        if not self.stale:
            return self.e.buf.stats.cpu().numpy()
        if self._host is None:
            self._host = torch.empty_like(self.e.buf.stats, device="cpu").pin_memory()
            self._copied = torch.cuda.Event()
            now = self.last.copy()   # nothing copied yet: no new evidence
        else:
            self._copied.synchronize()   # recorded an interval ago: long complete
            now = self._host.numpy().astype(np.int64)
        self._host.copy_(self.e.buf.stats, non_blocking=True)
        self._copied.record()
        return now

    def step(self) -> int:
        now = self._counters()
        pa = -1.0 if self.prior_alpha == "pooled" else float(self.prior_alpha)
        if self.round_costs is not None:
            k, self.last_prior = L.s3r_horizon_step_costs(now, self.last, self.acc, self.dec, self.k_max,
                                                          self.decay, self.round_costs, pa, self.prior_weight)
        else:
            k, self.last_prior = L.s3r_horizon_step(now, self.last, self.acc, self.dec, self.k_max, self.decay,
                                                    self.c_draft, self.c_verify, pa, self.prior_weight)
        self.e.set_k(k)
        self.history.append(k)
        return k
