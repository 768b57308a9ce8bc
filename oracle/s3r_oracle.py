"""Plain, slow CPU oracle of one S3R draft+verify round, in float64 (numpy).

TEST INFRASTRUCTURE ONLY. The CUDA library never imports or calls this module; it exists
so the tests, the smoke check and the benchmark's CPU baseline can check and time the
GPU path against a definition that a reader can compare with the pages by eye.

Sources (cited by page title and section):
  [News]      "Long-context RL training stops waiting on autoregressive rollouts: sparse
              self-drafting plus full-attention verification lifts throughput 1.39x"
              (ai4snews summary), sections Interpretation and Perspective.
  [Listing]   "S^3R: Fast and Faithful RL Rollouts via Self-Sparse Speculative Decoding"
              (paper listing), Abstract, Table 1, appendix Tables 4-7.
  [Explainer] "S3R - Self-sparse speculative rollouts for RL - What does it mean?",
              Jargon list, walkthrough, and "Where it earns its keep".
  [Wispaper]  Chinese summary of the same paper, sections on sparse drafting / dense
              verification and on per-position acceptance.

The pages print no formulas for this path, so each step below is the plain textbook
definition of what the pages name, with the readings listed at the step:
  * attention logits s_j = <q, k_j> / sqrt(d), softmax over the visible positions;
  * the score of a cached position is the softmax probability the last dense verify
    gave it, summed over the query heads that share its KV head and over all k+1 rows
    of the verified block (rows after the first rejection included: the scores are
    taken before sampling decides);
  * the sparse set of a request / KV head holds n = ceil(L * s) positions, s in basis
    points (integer ceil): the newest min(W, L) positions plus the highest-scored
    remaining ones, ties to the lower position, sorted ascending;
  * exact speculative sampling in the standard form (accept with probability
    min(1, p/q), else draw from the normalised residual max(0, p - q); a bonus draw
    from the last target row when every draft is accepted);
  * uniforms from Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
    as easy as 1, 2, 3", SC'11) keyed by the sampling seed, counter (position, request,
    stream, 0), u = (word0 >> 8) * 2^-24.

Parity pinned by tests/test_oracle_*.py (brute force, closed forms, invariants,
published known-answer vectors, distribution tests); nothing here is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

PAGE_SIZE = 16

# ----------------------------------------------------------------------------------------
# Paged KV layout: position j of a request lives in page page_table[j // 16], slot j % 16,
# and a pool is indexed [page][kv_head][slot][dim].  [News] Perspective (complete
# historical KV kept for the dense verify); [Explainer] walkthrough ("pages").
# ----------------------------------------------------------------------------------------


def gather_positions(pool, page_table_row, kv_head: int, positions) -> np.ndarray:
    """K or V rows [n][d] (float64) of one request / KV head at the given positions."""
    positions = np.asarray(positions, dtype=np.int64)
    pages = np.asarray(page_table_row, dtype=np.int64)[positions // PAGE_SIZE]
    if np.any(pages < 0):
        raise IndexError("position maps to an unallocated page")
    return np.asarray(pool[pages, kv_head, positions % PAGE_SIZE], dtype=np.float64)


# ----------------------------------------------------------------------------------------
# O1 + O2: dense attention of the verify block, with score capture.
# [News] Interpretation: verification recomputes the proposed block against the complete
# historical KV; drafting picks KV entries "using attention scores".
# [Explainer] walkthrough: the top-scoring entries come from the verifier's last attention
# pass and are refreshed after every round.
# ----------------------------------------------------------------------------------------


def attention_row(q: np.ndarray, K: np.ndarray, V: np.ndarray):
    """Softmax attention of one query row over the rows of K/V (all visible).

    Returns (output [d], log-sum-exp of the logits, probabilities [n], logits [n]).
    """
    d = q.shape[-1]
    s = (K @ q) / math.sqrt(d)
    m = s.max()
    e = np.exp(s - m)
    z = e.sum()
    p = e / z
    return p @ V, m + math.log(z), p, s


def verify_attention(q_block: np.ndarray, K: np.ndarray, V: np.ndarray, L: int):
    """Dense verify of a block of T = k+1 rows at positions L .. L+k.

    q_block [T][H_q][d]; K, V [H_kv][>= L+T][d] hold the complete context, block included.
    Row t attends positions 0 .. L+t (causal inside the block). Query head h uses KV head
    h // G (contiguous grouping, G = H_q / H_kv).

    Returns out [T][H_q][d], lse [T][H_q], sigma [H_kv][L+T] (scores: probabilities summed
    over the G heads of the group and over all T rows) and logits [H_kv][G*T][L+T]
    (row index t*G + g; -inf where masked).
    """
    T, Hq, d = q_block.shape
    Hkv = K.shape[0]
    G = Hq // Hkv
    n = L + T
    out = np.zeros((T, Hq, d))
    lse = np.zeros((T, Hq))
    sigma = np.zeros((Hkv, n))
    logits = np.full((Hkv, G * T, n), -np.inf)
    for h in range(Hq):
        kvh = h // G
        g = h % G
        for t in range(T):
            vis = L + t + 1
            o, l, p, s = attention_row(q_block[t, h], K[kvh, :vis], V[kvh, :vis])
            out[t, h] = o
            lse[t, h] = l
            sigma[kvh, :vis] += p
            logits[kvh, t * G + g, :vis] = s
    return out, lse, sigma, logits


def scores_from_logits(logits: np.ndarray, lse: np.ndarray) -> np.ndarray:
    """sigma_j = sum over rows of exp(logit[row, j] - lse[row]) (rows of one KV head).

    logits [R][n] with -inf where a row does not see position j; lse [R].
    """
    return np.exp(logits - lse[:, None]).sum(axis=0)


# ----------------------------------------------------------------------------------------
# O3: sparse KV selection.
# [Explainer] Jargon "sparse attention budget": a token may read a fraction s of the cached
# positions (s = 0.05): the newest positions plus those the verifier attended to most.
# [Explainer] walkthrough: refreshed after every round. Readings: the window counts inside
# the budget; n = ceil(L * s) in integer basis points; if n < W only the window is kept;
# ties go to the lower position; output ascending.
# ----------------------------------------------------------------------------------------


def budget_count(L: int, budget_bp: int, window: int):
    """(n, W') for committed length L: n = clamp(ceil(L*bp/1e4), W', L), W' = min(W, L)."""
    n = -(-(L * budget_bp) // 10000)
    w = min(window, L)
    return min(max(n, w), L), w


def select_positions(sigma: np.ndarray, L: int, budget_bp: int, window: int) -> np.ndarray:
    """Sorted positions of the sparse set for committed length L.

    sigma holds at least the scores of positions 0 .. L-W'-1 (the non-window positions).
    The top M = n - W' non-window positions by score are found by their threshold: the
    M-th largest score T; every position scoring above T is taken, then positions scoring
    exactly T in increasing order until M are taken.
    """
    n, w = budget_count(L, budget_bp, window)
    m = n - w
    nonwin = L - w
    chosen = np.zeros(0, dtype=np.int64)
    if m > 0:
        s = np.asarray(sigma[:nonwin], dtype=np.float64)
        thr = np.sort(s)[::-1][m - 1]
        above = np.nonzero(s > thr)[0]
        ties = np.nonzero(s == thr)[0][: m - above.size]
        chosen = np.sort(np.concatenate([above, ties]))
    return np.concatenate([chosen, np.arange(nonwin, L)]).astype(np.int32)


def selection_margin_cases(sigma: np.ndarray, L: int, budget_bp: int, window: int,
                           rel: float = 1e-5) -> np.ndarray:
    """Non-window positions whose score lies within rel * threshold of the threshold.

    Selections at these positions may differ between two correct implementations whose
    scores differ by rounding; they are counted, not compared.
    """
    n, w = budget_count(L, budget_bp, window)
    m = n - w
    if m <= 0:
        return np.zeros(0, dtype=np.int64)
    s = np.asarray(sigma[: L - w], dtype=np.float64)
    thr = np.sort(s)[::-1][m - 1]
    return np.nonzero(np.abs(s - thr) <= rel * thr)[0]


# ----------------------------------------------------------------------------------------
# O3p: page-granular selection (the second reading of the selection rule).
# [Explainer] walkthrough: the draft reads the newest window plus the top-scoring *pages*
# from the verifier's last attention pass (the Jargon entry says positions). Reading: a
# page's score is the sum of its positions' scores, added in position order in the dtype of
# the scores given; the pages holding the W' newest positions are always kept (whole, so up
# to 15 older positions ride along); the budget is ceil(n / P) pages for the token budget n
# of budget_count and page size P; the remaining pages are the top-scoring pages wholly
# before the window, ties to the lower page; the set is every position of the chosen pages
# below L, ascending. With P = 1 this is select_positions.
# ----------------------------------------------------------------------------------------


def page_scores(sigma: np.ndarray, npages: int, page: int) -> np.ndarray:
    """Score of pages 0 .. npages-1: sigma[P*q] + sigma[P*q+1] + ... in that order, each add
    rounded to sigma's dtype (float32 scores give float32 sums)."""
    s = np.asarray(sigma)
    if npages == 0:
        return np.zeros(0, dtype=s.dtype)
    blocks = s[: npages * page].reshape(npages, page)
    acc = blocks[:, 0].copy()
    for t in range(1, page):
        acc = acc + blocks[:, t]
    return acc


def select_pages(sigma: np.ndarray, L: int, budget_bp: int, window: int, page: int = 16) -> np.ndarray:
    """Sorted positions of the page-granular sparse set for committed length L."""
    n, w = budget_count(L, budget_bp, window)
    first_win = (L - w) // page                  # first page holding a window position
    win_pages = -(-L // page) - first_win
    m = max(-(-n // page) - win_pages, 0)        # candidate pages to choose
    chosen = np.zeros(0, dtype=np.int64)
    if m > 0:
        ps = page_scores(sigma, first_win, page)
        thr = np.sort(ps)[::-1][m - 1]
        above = np.nonzero(ps > thr)[0]
        ties = np.nonzero(ps == thr)[0][: m - above.size]
        chosen = np.sort(np.concatenate([above, ties]))
    pos = (chosen[:, None] * page + np.arange(page)[None, :]).reshape(-1)
    return np.concatenate([pos, np.arange(first_win * page, L)]).astype(np.int32)


def page_selection_margin_cases(sigma: np.ndarray, L: int, budget_bp: int, window: int,
                                page: int = 16, rel: float = 1e-5) -> np.ndarray:
    """Candidate pages whose score lies within rel * threshold of the threshold (their
    selection may differ between two correct implementations; counted, not compared)."""
    n, w = budget_count(L, budget_bp, window)
    first_win = (L - w) // page
    m = max(-(-n // page) - (-(-L // page) - first_win), 0)
    if m <= 0:
        return np.zeros(0, dtype=np.int64)
    ps = np.asarray(page_scores(sigma, first_win, page), dtype=np.float64)
    thr = np.sort(ps)[::-1][m - 1]
    return np.nonzero(np.abs(ps - thr) <= rel * thr)[0]


# ----------------------------------------------------------------------------------------
# O4: sparse self-draft attention.
# [News] Interpretation and [Explainer] "How is this different": the draft uses the same
# weights, reading only the selected subset of the KV cache. Draft step i (token at
# position L+i) attends the selected set S plus the block positions L .. L+i written so
# far in this round; S stays fixed for the whole round.
# ----------------------------------------------------------------------------------------


def draft_positions(sel: np.ndarray, L: int, i: int) -> np.ndarray:
    return np.concatenate([np.asarray(sel, dtype=np.int64), np.arange(L, L + i + 1)])


def sparse_draft_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, sel, L: int, i: int):
    """q [H_q][d]; K, V [H_kv][>= L+i+1][d]; sel[kvh] = sorted selected positions (< L).

    Returns out [H_q][d] and lse [H_q].
    """
    Hq, d = q.shape
    Hkv = K.shape[0]
    G = Hq // Hkv
    out = np.zeros((Hq, d))
    lse = np.zeros(Hq)
    for h in range(Hq):
        kvh = h // G
        a = draft_positions(sel[kvh], L, i)
        o, l, _, _ = attention_row(q[h], K[kvh, a], V[kvh, a])
        out[h] = o
        lse[h] = l
    return out, lse


# ----------------------------------------------------------------------------------------
# O5: Philox4x32-10 (Salmon et al., SC'11): ten rounds of two 32x32->64 multiplies with
# the round multipliers below, Weyl key bumps between rounds.
# ----------------------------------------------------------------------------------------

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
_MASK = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key) -> np.ndarray:
    """Philox4x32-10 block function. ctr [..., 4], key [..., 2] (uint32) -> [..., 4] uint32."""
    c = np.asarray(ctr, dtype=np.uint64) & _MASK
    k = np.asarray(key, dtype=np.uint64) & _MASK
    c0, c1, c2, c3 = (c[..., i].copy() for i in range(4))
    k0, k1 = k[..., 0].copy(), k[..., 1].copy()
    for rnd in range(10):
        if rnd:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK
        p0 = np.uint64(PHILOX_M0) * c0
        p1 = np.uint64(PHILOX_M1) * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


STREAM_DRAFT, STREAM_ACCEPT, STREAM_DRAW = 0, 1, 2


def uniform(seed: int, request, position, stream: int) -> np.ndarray:
    """u in [0, 1): 24 high bits of word 0 of Philox4x32-10(key=seed, ctr=(pos, r, stream, 0))."""
    request = np.asarray(request, dtype=np.uint64)
    position = np.asarray(position, dtype=np.uint64)
    request, position = np.broadcast_arrays(request, position)
    ctr = np.stack([position, request, np.full_like(position, stream),
                    np.zeros_like(position)], axis=-1)
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint64)
    w = philox4x32_10(ctr, np.broadcast_to(key, ctr.shape[:-1] + (2,)))
    return (w[..., 0] >> np.uint32(8)).astype(np.float64) * (2.0 ** -24)


# ----------------------------------------------------------------------------------------
# O6 + O7: sampling.
# [News] Interpretation and [Explainer] Jargon "exact speculative sampling": accept or draw
# from the residual distribution, so emitted tokens follow the dense policy. Temperature 1.
# Token at position L+j+1: draft row j gives q_j, target row j gives p_j.
# ----------------------------------------------------------------------------------------


def softmax64(logits) -> np.ndarray:
    x = np.asarray(logits, dtype=np.float64)
    e = np.exp(x - x.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def inverse_cdf(weights, u: float):
    """Smallest v with u * Z < C_v (C inclusive cumulative sum, Z its total).

    Returns (v, margin) where margin is the distance of u to the nearer of C_{v-1}/Z and
    C_v/Z. If rounding leaves no such v, the last index with non-zero weight is taken.
    """
    w = np.asarray(weights, dtype=np.float64)
    c = np.cumsum(w)
    z = c[-1]
    hits = np.nonzero(u * z < c)[0]
    v = int(hits[0]) if hits.size else int(np.nonzero(w > 0)[0][-1])
    lo = c[v - 1] / z if v > 0 else 0.0
    return v, min(u - lo, c[v] / z - u)


def draft_sample(q_logits_row, u: float):
    """Draft token ~ softmax(q_logits_row) by inverse CDF with uniform u."""
    return inverse_cdf(softmax64(q_logits_row), u)


def spec_sample_request(p_logits, q_logits, drafts, u_accept, u_draw):
    """Exact speculative sampling for one request, uniforms given.

    p_logits [k+1][V] (target rows 0..k), q_logits [k][V] (draft rows 0..k-1),
    drafts [k]; u_accept[j] decides draft j, u_draw[j] draws the token at row j.
    Draft j is accepted iff u_accept[j] * q_j(d_j) < p_j(d_j). At the first rejection the
    token comes from max(0, p_j - q_j) normalised (from p_j if that is all zero); when all
    k drafts pass, a bonus token comes from p_k.

    Returns (tokens [a+1], n_out = a+1, margins) with margins[j] = |u_accept[j] - p/q| for
    each decided draft and a final entry for the draw.
    """
    p = softmax64(p_logits)
    q = softmax64(q_logits) if len(q_logits) else np.zeros((0, p.shape[-1]))
    k = len(drafts)
    tokens, margins = [], []
    for j in range(k):
        d = int(drafts[j])
        pj, qj = p[j, d], q[j, d]
        margins.append(abs(u_accept[j] - pj / qj) if qj > 0 else math.inf)
        if u_accept[j] * qj < pj:
            tokens.append(d)
            continue
        resid = np.maximum(0.0, p[j] - q[j])
        c, mg = inverse_cdf(resid if resid.sum() > 0 else p[j], u_draw[j])
        tokens.append(c)
        margins.append(mg)
        return np.asarray(tokens, dtype=np.int32), len(tokens), np.asarray(margins)
    c, mg = inverse_cdf(p[k], u_draw[k])
    tokens.append(c)
    margins.append(mg)
    return np.asarray(tokens, dtype=np.int32), len(tokens), np.asarray(margins)


def spec_sample(p_logits, q_logits, drafts, seed: int, request: int, L: int):
    """spec_sample_request with the Philox uniforms of request r at committed length L."""
    k = len(drafts)
    pos = L + 1 + np.arange(k + 1)
    ua = uniform(seed, request, pos[:k], STREAM_ACCEPT)
    ud = uniform(seed, request, pos, STREAM_DRAW)
    return spec_sample_request(p_logits, q_logits, drafts, ua, ud)


# ----------------------------------------------------------------------------------------
# Greedy (temperature 0) mode. [Listing] Table 4 setting (component measurements decode
# greedily): the draft token is the draft row's argmax, a draft is kept while it equals the
# target row's argmax, the first mismatch is replaced by the target argmax, and when all k
# agree the bonus token is the last target row's argmax. Ties go to the lowest token id;
# NaN logits count as -inf.
# ----------------------------------------------------------------------------------------
def argmax_token(logits_row) -> int:
    x = np.asarray(logits_row, dtype=np.float64)
    x = np.where(np.isnan(x), -np.inf, x)
    return int(np.argmax(x))   # numpy returns the first (lowest) index of the maximum


def greedy_verify(p_logits, drafts):
    """Tokens emitted by greedy verification: (tokens [a+1], n_out = a+1)."""
    k = len(drafts)
    tokens = []
    for j in range(k):
        t = argmax_token(p_logits[j])
        if t == int(drafts[j]):
            tokens.append(t)
            continue
        tokens.append(t)
        return np.asarray(tokens, dtype=np.int32), len(tokens)
    tokens.append(argmax_token(p_logits[k]))
    return np.asarray(tokens, dtype=np.int32), len(tokens)


# ----------------------------------------------------------------------------------------
# O-round: one draft+verify round of one request, composed from the steps above.
# [Explainer] walkthrough: draft k tokens from the sparse set, check all at once with one
# full pass, keep the agreeing prefix, replace the first mismatch, drop the rest.
# [Explainer] Jargon "block efficiency": tokens emitted per round (tau = a + 1).
# ----------------------------------------------------------------------------------------


class RequestState:
    """Dense per-request copy of the cache (positions in order) and the round state.

    `dtype` is the attention arithmetic's type: float64 (the default) for every parity
    use; float32 only for the benchmark's timing of a float32 CPU variant (the samplers
    stay float64 either way)."""

    def __init__(self, K: np.ndarray, V: np.ndarray, L: int, sigma: np.ndarray | None = None,
                 dtype=np.float64):
        self.K = np.array(K, dtype=dtype)   # [H_kv][capacity][d]
        self.V = np.array(V, dtype=dtype)
        self.L = int(L)
        self.sigma = sigma                       # scores from the last dense pass

    def write(self, positions, k_rows, v_rows):
        for p, kr, vr in zip(positions, k_rows, v_rows):
            self.K[:, p] = kr
            self.V[:, p] = vr


def prefill_scores(state: RequestState, q_x, k_x, v_x):
    """Scores for round 0: a one-row dense pass of the pending token at position L."""
    state.write([state.L], [k_x], [v_x])
    _, lse, sigma, _ = verify_attention(np.asarray(q_x, state.K.dtype)[None], state.K, state.V, state.L)
    state.sigma = sigma
    return lse, sigma


def run_round(state: RequestState, request: int, seed: int, k: int, budget_bp: int,
              window: int, q_rows, k_rows, v_rows, draft_logits, target_logits, page: int = 1,
              greedy: bool = False, timings: dict | None = None):
    """One round for one request.

    q_rows [k+1][H_q][d], k_rows/v_rows [k+1][H_kv][d]: projections of the tokens at
    positions L .. L+k (identical in draft and verify). draft_logits [k][V] give q_j,
    target_logits [k+1][V] give p_j for the token at position L+j+1. page > 1 selects whole
    pages of that size (O3p) instead of positions; greedy drafts and verifies by argmax
    (temperature 0) and has no sampling margins. `timings`, if given, accumulates the wall
    seconds of each step (select, draft_attn, draft_sample, verify, spec_sample) for the
    benchmark's CPU baseline; it does not change what is computed.
    """
    import time
    clock = [time.perf_counter()]

    def lap(name):
        if timings is not None:
            now = time.perf_counter()
            timings[name] = timings.get(name, 0.0) + now - clock[0]
            clock[0] = now

    L = state.L
    Hkv = state.K.shape[0]
    q_rows = np.asarray(q_rows, state.K.dtype)
    if page > 1:
        sel = [select_pages(state.sigma[h], L, budget_bp, window, page) for h in range(Hkv)]
    else:
        sel = [select_positions(state.sigma[h], L, budget_bp, window) for h in range(Hkv)]
    lap("select")
    drafts, draft_out, draft_margin = [], [], []
    for i in range(k):
        state.write([L + i], [k_rows[i]], [v_rows[i]])
        o, _ = sparse_draft_attention(q_rows[i], state.K, state.V, sel, L, i)
        draft_out.append(o)
        lap("draft_attn")
        if greedy:
            tok, mg = argmax_token(draft_logits[i]), np.inf
        else:
            u0 = float(uniform(seed, request, L + i + 1, STREAM_DRAFT))
            tok, mg = draft_sample(draft_logits[i], u0)
        drafts.append(tok)
        draft_margin.append(mg)
        lap("draft_sample")
    state.write(list(range(L, L + k + 1)), k_rows, v_rows)
    v_out, lse, sigma, logits = verify_attention(q_rows, state.K, state.V, L)
    lap("verify")
    if greedy:
        tokens, n_out = greedy_verify(target_logits, drafts)
        margins = np.array([np.inf])
    else:
        tokens, n_out, margins = spec_sample(target_logits, draft_logits, drafts, seed, request, L)
    lap("spec_sample")
    state.sigma = sigma
    state.L = L + n_out
    return dict(sel=sel, drafts=np.asarray(drafts, np.int32), draft_out=np.asarray(draft_out),
                draft_margin=np.asarray(draft_margin), verify_out=v_out, lse=lse, sigma=sigma,
                logits=logits, tokens=tokens, n_out=n_out, margins=margins)


# ----------------------------------------------------------------------------------------
# Round accounting. [Explainer] "Where it earns its keep": a round costs k sparse steps
# plus one dense pass and must emit more tokens than it costs. [Listing] Table 7: the
# break-even acceptance under sequential stage accounting for k drafts.
# ----------------------------------------------------------------------------------------


def expected_tau(alpha) -> float:
    """E[tokens per round] = 1 + sum_i prod_{j<=i} alpha_j for per-position acceptances."""
    tau, run = 1.0, 1.0
    for a in alpha:
        run *= a
        tau += run
    return tau


# ----------------------------------------------------------------------------------------
# O-horizon: adaptive draft length.
# [Wispaper] position-dependent acceptance: acceptance falls with the draft position and
# over training, and the authors propose shortening the draft horizon when the later
# positions' acceptance deteriorates (left to future work). [Listing] Table 7 prices a
# round under sequential stage accounting as k draft steps plus one verify (6 T_q + T_V at
# k = 6). Reading: estimate each position's acceptance from the counts so far, smoothed
# toward a prior, alpha_j = (accepted_j + w * alpha0) / (decided_j + w); take the k in
# [1, k_max] with the most expected tokens per unit round cost,
# expected_tau(alpha_1..alpha_k) / (k * c_draft + c_verify), the smallest k on ties.
# ----------------------------------------------------------------------------------------


def acceptance_estimate(accepted, decided, prior_alpha: float, prior_weight: float):
    """Smoothed per-position acceptance (a_j + w alpha0) / (d_j + w); the prior alone for a
    position never decided (w > 0)."""
    a = [float(x) for x in accepted]
    d = [float(x) for x in decided]
    return [(a[j] + prior_weight * prior_alpha) / (d[j] + prior_weight) for j in range(len(a))]


def choose_horizon(accepted, decided, c_draft: float, c_verify: float, k_max: int,
                   prior_alpha: float = 0.5, prior_weight: float = 4.0) -> int:
    """Draft length for the next rounds (see the block comment above)."""
    alpha = acceptance_estimate(accepted[:k_max], decided[:k_max], prior_alpha, prior_weight)
    best_k, best = 1, -1.0
    for k in range(1, k_max + 1):
        rate = expected_tau(alpha[:k]) / (k * c_draft + c_verify)
        if rate > best:
            best_k, best = k, rate
    return best_k


def choose_horizon_costs(accepted, decided, round_cost, k_max: int, prior_alpha: float = 0.5,
                         prior_weight: float = 4.0) -> int:
    """The same choice with the cost of a round measured per draft length (round_cost[k-1]
    for length k) instead of the line k * c_draft + c_verify: the k with the most expected
    tokens per unit cost, the smallest k on ties."""
    alpha = acceptance_estimate(accepted[:k_max], decided[:k_max], prior_alpha, prior_weight)
    best_k, best = 1, -1.0
    for k in range(1, k_max + 1):
        rate = expected_tau(alpha[:k]) / float(round_cost[k - 1])
        if rate > best:
            best_k, best = k, rate
    return best_k


def horizon_update(acc, dec, accepted_new, decided_new, decay: float):
    """Decayed counts per position: acc_j <- decay * acc_j + accepted_new_j, the same for the
    decided counts (positions that stop being drafted fade toward the prior)."""
    acc = [decay * float(a) + float(n) for a, n in zip(acc, accepted_new)]
    dec = [decay * float(d) + float(n) for d, n in zip(dec, decided_new)]
    return acc, dec


def pooled_prior(acc, dec, k_max: int, default: float = 0.5) -> float:
    """Acceptance pooled over positions 1..k_max (the plain expectation for a position with
    no evidence of its own): sum of accepted / sum of decided, summed in position order;
    `default` when nothing was decided."""
    sa, sd = 0.0, 0.0
    for j in range(k_max):
        sa += float(acc[j])
        sd += float(dec[j])
    return sa / sd if sd > 0 else default


def horizon_step(acc, dec, accepted_new, decided_new, decay: float, c_draft: float,
                 c_verify: float, k_max: int, prior_alpha=None, prior_weight: float = 4.0):
    """One decision of the adaptive draft length: decay the counts, add the new ones, take
    the prior (pooled when prior_alpha is None) and choose k. Returns (acc, dec, prior, k)."""
    acc, dec = horizon_update(acc, dec, accepted_new, decided_new, decay)
    prior = pooled_prior(acc, dec, k_max) if prior_alpha is None else float(prior_alpha)
    return acc, dec, prior, choose_horizon(acc[:k_max], dec[:k_max], c_draft, c_verify, k_max, prior,
                                           prior_weight)


def horizon_step_costs(acc, dec, accepted_new, decided_new, decay: float, round_cost, k_max: int,
                       prior_alpha=None, prior_weight: float = 4.0):
    """horizon_step choosing with per-length round costs. Returns (acc, dec, prior, k)."""
    acc, dec = horizon_update(acc, dec, accepted_new, decided_new, decay)
    prior = pooled_prior(acc, dec, k_max) if prior_alpha is None else float(prior_alpha)
    return acc, dec, prior, choose_horizon_costs(acc[:k_max], dec[:k_max], round_cost, k_max, prior,
                                                 prior_weight)


def break_even_acceptance(total_ms: float, ar_ms: float, k: int) -> float:
    """Acceptance at which a round (draft + verify = total) costs as much per token as AR.

    A round emits 1 + alpha*k tokens on average under a flat per-position acceptance;
    AR spends ar_ms on k+1 tokens, so break-even is (1 + alpha*k)/(k+1) * ar = total.
    """
    return ((k + 1) * total_ms / ar_ms - 1.0) / k
