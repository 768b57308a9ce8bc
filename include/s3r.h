/*
 * s3r.h - C ABI of libs3r.so: the per-round hot path of Self-Sparse Speculative Rollouts
 * (S3R) over a paged bf16 GQA KV cache, as hand-written CUDA kernels for sm_100a (B200).
 *
 * Sources (by page title and section):
 *   [News]      "Long-context RL training stops waiting on autoregressive rollouts: sparse
 *               self-drafting plus full-attention verification lifts throughput 1.39x",
 *               Interpretation and Perspective.
 *   [Listing]   "S^3R: Fast and Faithful RL Rollouts via Self-Sparse Speculative Decoding",
 *               Abstract; appendix Tables 4-7.
 *   [Explainer] "S3R - Self-sparse speculative rollouts for RL - What does it mean?",
 *               Jargon, walkthrough, "Where it earns its keep".
 *
 * One round of one request with committed length L and pending token x at position L:
 *   s3r_select_kv          sparse set S (n = ceil(s*L) positions) from the last verify's scores
 *   s3r_select_kv_pages    the same budget in whole 16-position pages
 *   k x s3r_sparse_draft_attn + s3r_draft_sample     draft tokens d_1..d_k
 *   s3r_verify_attn        dense attention of the k+1 rows at L..L+k, with score capture
 *   s3r_spec_sample        exact speculative sampling -> a accepted drafts + 1 token
 *   s3r_commit             L <- L + a + 1, acceptance counters
 *   s3r_choose_horizon     (host) draft length for the next rounds from those counters
 *   s3r_sched_simulate     (host) KV-aware AIMD admission of requests to a replica
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless it is marked
 *     "host". The library keeps no pointer after a call returns and allocates no memory.
 *   - Every call is asynchronous on the given stream (NULL = legacy default stream) and
 *     returns an s3r_status. Arguments are validated on the host before anything is
 *     launched; a non-OK status means nothing was launched.
 *   - Faults the host cannot see (a page id outside the pool, a selected index >= L, a
 *     context longer than the page table, a non-finite logit, an expired wait) are
 *     recorded in the workspace's error word as bit (1 << S3R_ERR_*) and the offending
 *     access is skipped; kernels never trap. s3r_get_error() reads and clears the word.
 *   - KV pools: bf16 [num_pages][num_kv_heads][16][head_dim]; head_dim is 64 or 128.
 *     Query head h reads KV head h / G, G = num_q_heads / num_kv_heads <= 8.
 *   - Requests: a launch covers `batch` requests; with req_ids == NULL they are requests
 *     0..batch-1, else req_ids[0..batch-1], which must be distinct and in [0, num_requests)
 *     (every kernel checks the range on the device: an id outside it sets
 *     S3R_ERR_DEVICE_BOUNDS and that request is skipped; s3r_commit, which has no error
 *     word, skips it). Every per-request array is indexed
 *     by the request id (size num_requests), so a launch can cover a subset of a larger
 *     batch (mixed round phases).
 *     Attention and selection calls cover at most 65535 requests per launch.
 *   - Page table: int32 [num_requests][max_pages_per_req]; position j of request r is
 *     slot j % 16 of page page_table[r][j / 16]. capacity = 16 * max_pages_per_req.
 *   - A workspace serves one stream at a time. It must be zeroed once by
 *     s3r_workspace_init before first use; every call leaves it ready for the next.
 */
#ifndef S3R_H_
#define S3R_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define S3R_API __attribute__((visibility("default")))
#else
#define S3R_API
#endif

typedef struct CUstream_st* s3r_stream_t; /* same handle as cudaStream_t */

typedef enum {
  S3R_OK = 0,
  S3R_ERR_INVALID_ARG = 1,   /* a NULL/misaligned pointer or a size out of range */
  S3R_ERR_UNSUPPORTED = 2,   /* head_dim, page size, group or k outside what is built */
  S3R_ERR_CUDA = 3,          /* a CUDA runtime call failed (launch, copy, attribute) */
  S3R_ERR_WORKSPACE = 4,     /* workspace NULL, misaligned or smaller than needed */
  S3R_ERR_DEVICE_BOUNDS = 5, /* device: page id / index / length outside its range */
  S3R_ERR_NONFINITE = 6,     /* device: NaN or Inf in logits or scores */
  S3R_ERR_TIMEOUT = 7        /* device: a bounded wait on a copy expired */
} s3r_status;

#define S3R_PAGE_SIZE 16
#define S3R_MAX_K 8          /* draft length k <= 8 */
#define S3R_MAX_GROUP 8      /* query heads per KV head */
#define S3R_MAX_ROWS 64      /* G * (k + 1) rows of one KV head in a verify */

typedef struct {
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;          /* 64 or 128 */
  int32_t page_size;         /* must be 16 */
  int64_t num_pages;
  void* k_pool;              /* bf16 [num_pages][num_kv_heads][16][head_dim], 16-byte aligned */
  void* v_pool;              /* same layout */
} s3r_kv_cache;

typedef struct {
  int32_t batch;             /* requests covered by this launch (0 = nothing to do) */
  int32_t num_requests;      /* size of every per-request array */
  const int32_t* req_ids;    /* [batch] request ids, or NULL for 0..batch-1 */
  const int32_t* seq_lens;   /* [num_requests] committed length L per request */
  const int32_t* page_table; /* [num_requests][max_pages_per_req] */
  int32_t max_pages_per_req;
} s3r_batch;

/* Bytes of workspace that every call below needs for a cache with this shape, up to
 * num_requests requests, page tables of max_pages_per_req pages, draft length <= max_k,
 * vocabularies <= vocab and selections of <= sel_stride positions. Pure host function. */
S3R_API size_t s3r_workspace_size(const s3r_kv_cache* cache, int32_t num_requests,
                          int32_t max_pages_per_req, int32_t max_k, int32_t vocab,
                          int32_t sel_stride);

/* Zero a workspace (256-byte aligned device buffer of ws_bytes bytes). */
S3R_API int s3r_workspace_init(void* ws, size_t ws_bytes, s3r_stream_t stream);

/* Dense verify attention with score capture ([News] Interpretation: verification recomputes
 * the proposed block against the complete historical KV; [Explainer] walkthrough: the
 * sparse set is refreshed from the verifier's last attention pass).
 *   k          draft length; the block has T = k+1 rows at positions L..L+k (0 <= k <= 8;
 *              k = 0 is the one-row pass of a prefill's last token).
 *   q          bf16 [num_requests][T][H_q][d]; row t of head h attends positions 0..L+t.
 *   k_new,v_new bf16 [num_requests][T][H_kv][d]: K/V of the block; written into the pages
 *              of positions L..L+k (which must be allocated) and used for the block.
 *   out        bf16 [num_requests][T][H_q][d], softmax(q K^T / sqrt(d)) V rounded once.
 *   lse        fp32 [num_requests][T][H_q], natural-log log-sum-exp of the logits.
 *   score_logits fp32 [num_requests][H_kv][G*T][capacity] or NULL: logit q.k/sqrt(d) of
 *              row t*G+g of each KV head at every committed position j < L, the positions
 *              of one row contiguous (entries at j >= L are not written). With lse it
 *              defines the scores of s3r_select_kv.
 * q, k_new, v_new, out and score_logits must be 16-byte aligned, lse 4-byte aligned
 * (S3R_ERR_INVALID_ARG otherwise). Needs L + T <= capacity (device check). */
S3R_API int s3r_verify_attn(const s3r_kv_cache* cache, const s3r_batch* batch, int32_t k,
                    const void* q, const void* k_new, const void* v_new, void* out,
                    float* lse, float* score_logits, void* ws, size_t ws_bytes,
                    s3r_stream_t stream);

/* Sparse KV selection ([Explainer] Jargon, sparse attention budget: a fraction s of the
 * cached positions, the newest ones plus those the verifier attended to most).
 * For request r at committed length L (seq_lens, already advanced by s3r_commit) and KV
 * head h: W' = min(window, L), n = clamp(ceil(L * budget_bp / 10000), W', L), and the set
 * is the W' newest positions plus the n - W' positions j < L - W' of highest score
 *   sigma_j = sum over the G*(k_prev+1) rows of exp(score_logits[row][j] - lse[row]),
 * ties to the lower j, written ascending to sel_idx[r][h][0..n-1]; sel_count[r][h] = n.
 *   score_logits, lse  as written by the previous s3r_verify_attn with k = k_prev
 *              (score_logits 16-byte aligned). The exponentials are formed as
 *              2^(x log2(e) - lse log2(e)) in fp32 (relative error about 1e-6).
 *   Two launches: the scores of every (request, KV head) into the workspace (4 bytes per
 *   position of the page-table capacity, counted by s3r_workspace_size), then the selection.
 *   sel_idx    int32 [num_requests][H_kv][sel_stride]; n > sel_stride is a device bounds
 *              error. sel_count int32 [num_requests][H_kv].
 * Needs 1 <= budget_bp <= 10000 and window >= k_prev + 1 (so that every scored non-window
 * position is committed), L - W' <= 49152. */
S3R_API int s3r_select_kv(const s3r_kv_cache* cache, const s3r_batch* batch, const float* score_logits,
                  const float* lse, int32_t k_prev, int32_t budget_bp, int32_t window,
                  int32_t* sel_idx, int32_t sel_stride, int32_t* sel_count, void* ws,
                  size_t ws_bytes, s3r_stream_t stream);

/* The scores s3r_select_kv orders positions by, on their own: for request r (committed length
 * L at this call) and KV head h, scores[r][h][j] = sum over the G*(k_prev+1) rows of
 * exp(logit - lse) for every j < L, the same fp32 values s3r_select_kv computes.
 * s3r_select_from_scores on them makes the same selection as s3r_select_kv. The two halves
 * split where the round allows it: a selection at committed length L' (at most L + k_prev + 1,
 * fewer than W positions more) reads only j < L' - W < L, so these scores can be computed
 * as soon as the verify's logits and lse exist, while speculative sampling and the commit run
 * on another stream; only the ordering waits for the new lengths.
 *   scores  fp32 [num_requests][H_kv][score_stride], 16-byte aligned, score_stride a multiple
 *           of 4 and >= L (a longer context sets S3R_ERR_DEVICE_BOUNDS); entries j >= L are
 *           not written. Uses only the workspace's error word. */
S3R_API int s3r_position_scores(const s3r_kv_cache* cache, const s3r_batch* batch,
                        const float* score_logits, const float* lse, int32_t k_prev,
                        float* scores, int32_t score_stride, void* ws, size_t ws_bytes,
                        s3r_stream_t stream);

/* The same selection from caller-given scores: scores fp32 [num_requests][H_kv][score_stride],
 * sigma_j = scores[r][h][j] (any finite float; order by value, ties to the lower j). */
S3R_API int s3r_select_from_scores(const s3r_kv_cache* cache, const s3r_batch* batch,
                           const float* scores, int32_t score_stride, int32_t budget_bp,
                           int32_t window, int32_t* sel_idx, int32_t sel_stride,
                           int32_t* sel_count, void* ws, size_t ws_bytes, s3r_stream_t stream);

/* Page-granular selection ([Explainer] walkthrough: the newest window plus the top-scoring
 * pages from the verifier's last attention pass). The units are the 16-position pages
 * wholly before the window, page q scored by sigma_16q + sigma_16q+1 + ... + sigma_16q+15
 * added in that order in fp32 (one rounding per add), sigma_j as for s3r_select_kv; the
 * pages that hold any of the W' newest positions are always kept, whole; the budget is
 * ceil(n / 16) pages in all (never fewer than the window's), the rest the highest-scored
 * candidate pages, ties to the lower page. Every position below L of a chosen page is
 * written, ascending: sel_count = 16 * (chosen candidate pages) + (L - 16 * first window
 * page) <= n + 15, so sel_stride must hold n + 15 positions (a larger count is a device
 * bounds error). Arguments, launches, workspace and errors as s3r_select_kv; the set is a
 * list of positions, so s3r_sparse_draft_attn reads it unchanged (whole pages are 4 KB
 * contiguous runs at d = 128). Needs (L - W') / 16 <= 49152. */
S3R_API int s3r_select_kv_pages(const s3r_kv_cache* cache, const s3r_batch* batch,
                        const float* score_logits, const float* lse, int32_t k_prev,
                        int32_t budget_bp, int32_t window, int32_t* sel_idx, int32_t sel_stride,
                        int32_t* sel_count, void* ws, size_t ws_bytes, s3r_stream_t stream);

/* Page-granular selection from caller-given scores (layout as s3r_select_from_scores; a
 * non-finite score in a page makes that page's score -inf and sets S3R_ERR_NONFINITE). */
S3R_API int s3r_select_pages_from_scores(const s3r_kv_cache* cache, const s3r_batch* batch,
                                 const float* scores, int32_t score_stride, int32_t budget_bp,
                                 int32_t window, int32_t* sel_idx, int32_t sel_stride,
                                 int32_t* sel_count, void* ws, size_t ws_bytes,
                                 s3r_stream_t stream);

/* Sparse self-draft attention ([News] Interpretation; [Explainer] "How is this different":
 * the same weights reading a sparse subset of the KV cache). Draft step i = draft_step[r]
 * handles the token at position L+i: its K/V (k_new, v_new) are written to that position's
 * page, and its query rows attend S (sel_idx[r][h][0..n-1], every index < L) plus the block
 * positions L..L+i (the earlier ones written by the earlier steps of the round).
 *   q      bf16, request r's [H_q][d] rows at q + r * q_stride (elements; 0 means H_q * d)
 *   k_new, v_new bf16, request r's [H_kv][d] rows at k_new + r * kv_stride (0 means H_kv * d)
 *          (strides let a caller pass step i of a [num_requests][k+1][...] block in place)
 *   out    bf16 [num_requests][H_q][d];  lse fp32 [num_requests][H_q] or NULL. */
S3R_API int s3r_sparse_draft_attn(const s3r_kv_cache* cache, const s3r_batch* batch,
                          const int32_t* draft_step, const void* q, int32_t q_stride,
                          const void* k_new, const void* v_new, int32_t kv_stride,
                          const int32_t* sel_idx, int32_t sel_stride,
                          const int32_t* sel_count, void* out, float* lse, void* ws,
                          size_t ws_bytes, s3r_stream_t stream);

/* Normaliser of one row of logits x: max = max_v x_v and sum = sum_v exp(x_v - max), so that
 * softmax(x)_v = exp(x_v - max) / sum (non-finite entries count as -inf). 16 bytes. */
typedef struct s3r_row_norm {
  float max;
  float reserved;
  double sum;
} s3r_row_norm;

/* Draft-token sampling (temperature 1). For request r at step i = draft_step[r]:
 * q_i = softmax(q_logits[r][i][0..vocab-1]); u = Philox4x32-10(key = seed,
 * counter = (L+i+1, r, 0, 0)) word 0 >> 8, times 2^-24; the token is the smallest v with
 * u * Z < C_v (C inclusive cumulative sum of exp(x - max), Z its total), written to
 * draft_tokens[r][i].  q_logits fp32 [num_requests][k][vocab]; draft_tokens int32
 * [num_requests][k]. margins (fp32 [num_requests][k], may be NULL) receives the draw's
 * distance to the nearer edge of the drawn token's cell, min(u - C_{v-1}/Z, C_v/Z - u),
 * as this call computed the sums: a draw with a margin below the rounding of those sums
 * may go either way in another correct implementation. q_norm (s3r_row_norm
 * [num_requests][k], may be NULL) receives the normaliser of row i that the draw used, so
 * that s3r_spec_sample can take it instead of streaming the row again. */
S3R_API int s3r_draft_sample(const s3r_batch* batch, const int32_t* draft_step, int32_t k,
                     const float* q_logits, int32_t vocab, uint64_t seed, int32_t* draft_tokens,
                     float* margins, s3r_row_norm* q_norm, void* ws, size_t ws_bytes,
                     s3r_stream_t stream);

/* s3r_draft_sample without a workspace. The paper has no counterpart: this is a
 * library convenience for callers that cannot hand the library device memory at the
 * point of the call: a host program that drives the library from plain C without an
 * allocator of its own, or a server that has given all free HBM to the KV pool and must
 * not allocate between rounds. Same arguments, arithmetic and outputs as
 * s3r_draft_sample (without margins), bit for bit; the scratch (arrival tickets, per-chunk
 * partials and sub-block sums) lives in a static device array inside the library, 8 KiB +
 * 3 MiB per device that loads the library, held until the process exits, so
 *   - num_requests <= S3R_NOALLOC_MAX_REQUESTS and vocab <= S3R_NOALLOC_MAX_VOCAB, else
 *     S3R_ERR_UNSUPPORTED with a message in s3r_last_error_message() and no launch;
 *   - err_word (device int32, caller-owned, zeroed by the caller before first use)
 *     receives the device-side status bits that the workspace's error word would get;
 *   - the first call on a device (the current device) looks the array's device address
 *     up (cudaGetSymbolAddress), so it belongs before any stream capture begins. Every
 *     call then clears the tickets of its num_requests requests with a cudaMemsetAsync on
 *     `stream` and launches one kernel on it;
 *   - the array is shared by every call on a device and keeps the last call's contents:
 *     two calls that may overlap on the GPU (other streams, other host threads) race on
 *     it and give wrong tokens; order them.
 * The library calls no allocation routine on this path. */
#define S3R_NOALLOC_MAX_REQUESTS 2048
#define S3R_NOALLOC_MAX_VOCAB 262144
S3R_API int s3r_draft_sample_noalloc(const s3r_batch* batch, const int32_t* draft_step,
                             int32_t k, const float* q_logits, int32_t vocab, uint64_t seed,
                             int32_t* draft_tokens, int32_t* err_word, s3r_stream_t stream);

/* Exact speculative sampling ([News] Interpretation; [Explainer] Jargon, exact speculative
 * sampling). p_j = softmax(p_logits[r][j]) (j = 0..k), q_j = softmax(q_logits[r][j])
 * (j < k) are the target / draft distributions of the token at position L+j+1.
 * Draft j is accepted iff u1 * q_j(d) < p_j(d), u1 from counter (L+j+1, r, 1, 0). At the
 * first rejection the token is drawn from max(0, p_j - q_j) normalised (from p_j if that is
 * all zero) with u2 from counter (L+j+1, r, 2, 0); if all k pass, from p_k with
 * counter (L+k+1, r, 2, 0).  out_tokens int32 [num_requests][k+1] receives the a accepted
 * drafts and the drawn token (entries after them untouched); n_out[r] = a + 1.
 * margins (fp32 [num_requests][k+1], may be NULL) receives the decisions' distances to
 * their boundaries, in decision order: |u1 - p_j(d)/q_j(d)| for each decided draft (the a
 * accepted ones and the rejected one, if any), then the draw's distance to the nearer edge
 * of the drawn token's cell (as for s3r_draft_sample); min(a + 1, k) + 1 entries are
 * written, the rest untouched. q_norm (s3r_row_norm [num_requests][k], may be NULL): the
 * normalisers of the q rows as s3r_draft_sample wrote them for these q_logits; with it the
 * q rows are read only at the drafted tokens and in the drawn row, not streamed whole
 * (13 -> 7 rows at k = 6). Without it they are computed here. */
S3R_API int s3r_spec_sample(const s3r_batch* batch, int32_t k, const float* p_logits,
                    const float* q_logits, const int32_t* draft_tokens, int32_t vocab,
                    uint64_t seed, int32_t* out_tokens, int32_t* n_out, float* margins,
                    const s3r_row_norm* q_norm, void* ws, size_t ws_bytes, s3r_stream_t stream);

/* Greedy (temperature 0) mode ([Listing] Table 4 setting: component measurements decode
 * greedily). s3r_draft_argmax: draft_tokens[r][i] = argmax of q_logits[r][i], i =
 * draft_step[r]. s3r_greedy_verify: with t_j = argmax of p_logits[r][j], drafts are kept
 * while draft_tokens[r][j] == t_j; out_tokens[r][0..a] = t_0..t_a (a = drafts kept, the
 * last one the replacement of the first mismatch or, when all k agree, the bonus t_k);
 * n_out[r] = a + 1. Ties go to the lowest token id; NaN logits count as -inf and set
 * S3R_ERR_NONFINITE. Layouts, workspace and limits as s3r_draft_sample / s3r_spec_sample;
 * one launch each. */
S3R_API int s3r_draft_argmax(const s3r_batch* batch, const int32_t* draft_step, int32_t k,
                     const float* q_logits, int32_t vocab, int32_t* draft_tokens, void* ws,
                     size_t ws_bytes, s3r_stream_t stream);
S3R_API int s3r_greedy_verify(const s3r_batch* batch, int32_t k, const float* p_logits,
                     const int32_t* draft_tokens, int32_t vocab, int32_t* out_tokens,
                     int32_t* n_out, void* ws, size_t ws_bytes, s3r_stream_t stream);

/* Commit a round ([Explainer] Jargon, block efficiency: tokens per round): for each
 * request of the batch, seq_lens[r] += n_out[r]. stats (int64, may be NULL) accumulates
 * [0] tokens emitted, [1] request-rounds, [2+j] drafts accepted at position j and
 * [2+S3R_MAX_K+j] drafts decided at position j (j < k); it has 2 + 2*S3R_MAX_K entries, laid
 * out alike whatever k, so rounds of different draft lengths count into the same array. */
S3R_API int s3r_commit(const s3r_batch* batch, int32_t k, const int32_t* n_out, int32_t* seq_lens,
               int64_t* stats, s3r_stream_t stream);

/* KV-aware admission of requests to one rollout replica ([News] summary: a KV-aware AIMD
 * scheduler adapts admission to limit repeated KV offloading and restoring while keeping
 * rollout parallelism; [Explainer] Jargon, AIMD scheduler: admit one more request when
 * GPU KV memory has room, halve the limit under pressure; [Explainer] "Where it earns its
 * keep": back off when pressure or the restore backlog grows; [Wispaper] "dense
 * verification still needs the complete KV cache": utilisation and the paused requests'
 * backlog drive it). HOST function, no device work: a discrete-event model of the
 * replica, one iteration per draft-and-verify round of all active requests:
 *   1. capacity C_t = capacity - pressure[t] pages (pressure may be NULL; t >= pressure_len:
 *      0), the injected memory-pressure events;
 *   2. each active request, in admission order, emits min(tau[r][j], left) tokens, j its
 *      own round count; finished requests free their pages;
 *   3. U = sum of ceil((prompt + generated) / 16) over active requests;
 *   4. while U > C_t the most recently admitted request is evicted to the FIFO paused
 *      queue (evict 0: its pages are offloaded to host memory, transferred += pages;
 *      evict 1: dropped, recomputed when restored);
 *   5. policy 0 (AIMD): cap = max(cap_min, cap / 2) if anything was evicted, U > u_high C_t
 *      or the paused requests' pages > b_high C_t; else cap = min(cap_max, cap + 1) if the
 *      cap binds (active >= cap) and U < u_low C_t. Policy 1 keeps cap = cap0;
 *   6. while active < cap: restore the head of the paused queue (transferred, or
 *      recomputed, += its pages), else admit the next new request (prefilled += its prompt
 *      pages), each only if U + pages <= C_t, else stop for this iteration;
 *   7. time += c0 + c_tok tokens_t + c_kv U + c_xfer transferred_t + c_rec recomputed_t +
 *      c_pre prefilled_t (in double, in that order).
 * The run ends when all requests are done, after max_iters, or when no progress is
 * possible (nothing active and the head of the queues cannot fit; result.stalled = 1).
 *   prompt_len, resp_len  host int32 [num_requests] (>= 0): prompt tokens, tokens to emit.
 *   tau                   host uint8 [num_requests][tau_stride]: tokens one round emits
 *                         for request r at its j-th active round (a run that needs more
 *                         than tau_stride rounds of one request is S3R_ERR_INVALID_ARG).
 *   pressure              host int32 [pressure_len] (0 <= pressure < capacity) or NULL.
 *   out                   totals; trace (host int32 [trace_cap][8], may be NULL): per
 *                         iteration cap, active, paused, U, transferred, recomputed,
 *                         prefilled, tokens, for the first trace_cap iterations.
 * S3R_ERR_INVALID_ARG for NULL inputs, sizes or parameters out of range. */
typedef struct {
  int32_t capacity;   /* GPU KV pages (16 tokens each) of the replica */
  int32_t policy;     /* 0 AIMD, 1 fixed cap */
  int32_t evict;      /* 0 offload to host memory, 1 recompute on restore */
  int32_t cap0, cap_min, cap_max;
  double u_low, u_high, b_high;
  double c0, c_tok, c_kv, c_xfer, c_rec, c_pre;
  int64_t max_iters;
} s3r_sched_config;

typedef struct {
  int64_t tokens, transferred, recomputed, prefilled, evictions, iterations;
  int32_t max_active, done, stalled, reserved;
  double time;
} s3r_sched_result;

S3R_API int s3r_sched_simulate(const s3r_sched_config* cfg, int32_t num_requests,
                       const int32_t* prompt_len, const int32_t* resp_len, const uint8_t* tau,
                       int64_t tau_stride, const int32_t* pressure, int64_t pressure_len,
                       s3r_sched_result* out, int32_t* trace, int64_t trace_cap);

/* Adaptive draft length ([Wispaper] position-dependent acceptance: shorten the draft
 * horizon when the later positions' acceptance falls; [Listing] Table 7: a round costs k
 * draft steps plus one verify). HOST function, no device work: with the smoothed
 * acceptance alpha_j = (accepted[j] + prior_weight * prior_alpha) / (decided[j] +
 * prior_weight) for positions j < k_max, writes to *k_out the k in [1, k_max] that
 * maximises (1 + sum_{i<=k} prod_{j<=i} alpha_j) / (k * c_draft + c_verify), the smallest
 * k on ties (all arithmetic in double, in that order).
 *   accepted, decided  host double [k_max]: counts per draft position (for instance the
 *                      stats of s3r_commit, possibly decayed over time); not kept.
 *   c_draft, c_verify  cost of one draft step and of the rest of a round (any unit, > 0).
 * S3R_ERR_INVALID_ARG for NULL pointers, k_max outside 1..S3R_MAX_K, a cost <= 0 or not
 * finite, prior_alpha outside [0, 1], prior_weight < 0, a negative count, or a position with
 * decided + prior_weight == 0. */
S3R_API int s3r_choose_horizon(const double* accepted, const double* decided, int32_t k_max,
                       double c_draft, double c_verify, double prior_alpha,
                       double prior_weight, int32_t* k_out);

/* s3r_choose_horizon with a measured cost per draft length instead of the line
 * k * c_draft + c_verify (HOST function, no device work): writes to *k_out the k in
 * [1, k_max] that maximises (1 + sum_{i<=k} prod_{j<=i} alpha_j) / round_cost[k-1], the
 * smallest k on ties, alpha_j as in s3r_choose_horizon (all arithmetic in double, in that
 * order). A round's cost need not grow linearly with k (the verify's row count steps, the
 * launches overlap), so costs taken per length can rank the lengths where a line cannot.
 *   round_cost  host double [k_max]: cost of one round at draft length k = 1..k_max (any
 *               unit, > 0); not kept.
 * S3R_ERR_INVALID_ARG for NULL pointers, a cost <= 0 or not finite, or any other argument
 * s3r_choose_horizon rejects. */
S3R_API int s3r_choose_horizon_costs(const double* accepted, const double* decided, int32_t k_max,
                             const double* round_cost, double prior_alpha, double prior_weight,
                             int32_t* k_out);

/* One decision of the adaptive draft length from the commit counters (HOST function, no
 * device work; [Wispaper] position-dependent acceptance). With the counters of s3r_commit
 * now and at the last decision (host int64 [2 + 2*S3R_MAX_K] each, that layout), for every
 * position j < S3R_MAX_K, in double:
 *   accepted[j] = decay * accepted[j] + (stats_now[2+j] - stats_last[2+j])
 *   decided[j]  = decay * decided[j]  + (stats_now[2+S3R_MAX_K+j] - stats_last[2+S3R_MAX_K+j])
 * then stats_last = stats_now; the prior is prior_alpha, or (prior_alpha < 0) the acceptance
 * pooled over positions j < k_max, sum accepted / sum decided added in position order (0.5
 * when nothing was decided), written to *prior_out (may be NULL); *k_out is then what
 * s3r_choose_horizon picks from accepted / decided [0, k_max) with that prior.
 *   accepted, decided  host double [S3R_MAX_K], the caller's decayed counts (start at 0).
 * S3R_ERR_INVALID_ARG for NULL pointers, decay outside [0, 1], a counter that went down, or
 * any argument s3r_choose_horizon rejects (then nothing is updated). */
S3R_API int s3r_horizon_step(const int64_t* stats_now, int64_t* stats_last, double* accepted,
                     double* decided, int32_t k_max, double decay, double c_draft,
                     double c_verify, double prior_alpha, double prior_weight,
                     double* prior_out, int32_t* k_out);

/* s3r_horizon_step choosing with s3r_choose_horizon_costs (round_cost host double [k_max]). */
S3R_API int s3r_horizon_step_costs(const int64_t* stats_now, int64_t* stats_last, double* accepted,
                           double* decided, int32_t k_max, double decay, const double* round_cost,
                           double prior_alpha, double prior_weight, double* prior_out, int32_t* k_out);

/* Philox4x32-10 words and uniforms for n counters (position[i], request[i], stream_id, 0)
 * under key = seed: words uint32 [n][4] (may be NULL), u fp32 [n] (may be NULL). */
S3R_API int s3r_philox(uint64_t seed, int32_t stream_id, const int32_t* request, const int32_t* position,
               int64_t n, uint32_t* words, float* u, s3r_stream_t stream);

/* Synchronise `stream`, copy the workspace error word to *device_error (host pointer; a
 * bitmask of (1 << S3R_ERR_*)) and clear it. Returns S3R_ERR_CUDA if the stream failed. */
S3R_API int s3r_get_error(void* ws, int32_t* device_error, s3r_stream_t stream);

/* Static text for a status code. */
S3R_API const char* s3r_status_string(int status);

/* Number of kernels this library has launched in the process (all calls, all streams). */
S3R_API uint64_t s3r_launch_count(void);

/* Choose the kernel behind s3r_verify_attn for later calls (process-wide): 0 = automatic
 * (the tcgen05 tensor-memory kernel for head_dim 128, G*(k+1) <= 64 rows padded to 16, 32
 * or 64; the mma.sync kernel for head_dim 64), 1 = always the mma.sync kernel. Both
 * compute the same function. */
S3R_API int s3r_set_verify_kernel(int32_t which);

/* Bound, in polls, on every wait of the tcgen05 verify kernel's roles for one another's
 * progress (process-wide, for later calls; 0 restores the default of 2^24 polls). A wait
 * that runs out sets S3R_ERR_TIMEOUT in the error word and the kernel winds down: each role
 * still waits, without this bound, for its own copies and tensor-core work in flight,
 * frees its tensor memory and returns, so the context stays usable. A diagnostic knob: a
 * small bound makes a correct launch time out on purpose. S3R_ERR_INVALID_ARG if polls < 0. */
S3R_API int s3r_set_wait_limit(int32_t polls);

/* Text of the CUDA error behind the last S3R_ERR_CUDA status returned on this thread
 * ("" if none). */
S3R_API const char* s3r_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* S3R_H_ */
