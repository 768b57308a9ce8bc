// The extern "C" boundary of libs3r.so: host-side validation, workspace carving, TMA
// descriptors and kernel launches. Nothing here allocates device memory.
#include <atomic>
#include <cstdio>
#include <cmath>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

using namespace s3r;

thread_local char g_last_error[256] = "";

namespace s3r {
int cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return S3R_OK;
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
  return S3R_ERR_CUDA;
}
}  // namespace s3r

namespace {

std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_verify_kernel{0};   // 0 auto, 1 CUDA-core mma.sync kernel
std::atomic<int> g_wait_limit{kWaitLimit};   // polls of the verify roles' waits on each other

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_cache(const s3r_kv_cache* c) {
  if (!c) return S3R_ERR_INVALID_ARG;
  if (c->page_size != S3R_PAGE_SIZE) return S3R_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return S3R_ERR_UNSUPPORTED;
  if (c->num_kv_heads <= 0 || c->num_q_heads <= 0 || c->num_q_heads % c->num_kv_heads)
    return S3R_ERR_INVALID_ARG;
  if (c->num_q_heads / c->num_kv_heads > S3R_MAX_GROUP) return S3R_ERR_UNSUPPORTED;
  if (c->num_kv_heads > kMaxKvHeads) return S3R_ERR_UNSUPPORTED;
  if (c->num_pages <= 0 || !c->k_pool || !c->v_pool) return S3R_ERR_INVALID_ARG;
  if (!aligned16(c->k_pool) || !aligned16(c->v_pool)) return S3R_ERR_INVALID_ARG;
  if ((int64_t)c->num_pages * c->num_kv_heads * S3R_PAGE_SIZE >= ((int64_t)1 << 31))
    return S3R_ERR_UNSUPPORTED;   // TMA row coordinate is a signed 32-bit integer
  return S3R_OK;
}

// need_pages: the call reads the page table (attention, selection); those kernels put the
// request in grid.y / grid.z, which limits a launch to 65535 requests.
int check_batch(const s3r_batch* b, bool need_pages) {
  if (!b) return S3R_ERR_INVALID_ARG;
  if (b->batch < 0 || b->num_requests < 0) return S3R_ERR_INVALID_ARG;
  if (b->batch == 0) return S3R_OK;
  if (!b->req_ids && b->batch > b->num_requests) return S3R_ERR_INVALID_ARG;
  if (!b->seq_lens || !aligned4(b->seq_lens)) return S3R_ERR_INVALID_ARG;
  if (b->req_ids && !aligned4(b->req_ids)) return S3R_ERR_INVALID_ARG;
  if (need_pages) {
    if (b->batch > 65535) return S3R_ERR_UNSUPPORTED;
    if (!b->page_table || !aligned4(b->page_table) || b->max_pages_per_req <= 0)
      return S3R_ERR_INVALID_ARG;
    if ((int64_t)b->max_pages_per_req * S3R_PAGE_SIZE >= ((int64_t)1 << 30))
      return S3R_ERR_UNSUPPORTED;
  }
  return S3R_OK;
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return S3R_ERR_WORKSPACE;
  if (ws_bytes < need) return S3R_ERR_WORKSPACE;
  return S3R_OK;
}

struct Carve {
  int* err;
  int* sched;
  int* tickets;
  uint8_t* part;
};

Carve carve(void* ws, int num_requests) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  Carve c;
  c.err = reinterpret_cast<int*>(b);
  c.sched = reinterpret_cast<int*>(b + kWsSchedOff);
  c.tickets = reinterpret_cast<int*>(b + kWsHeader);
  c.part = b + kWsHeader + ws_tickets_bytes(num_requests);
  return c;
}

size_t head_bytes(int num_requests) { return kWsHeader + ws_tickets_bytes(num_requests); }

int nvch_of(int vocab) { return (vocab + kVocabChunk - 1) / kVocabChunk; }

int finish(int st, int launches) {
  if (st == S3R_OK) g_launches.fetch_add((uint64_t)launches, std::memory_order_relaxed);
  return st;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D view of a pool: rows of head_dim bf16 (one per (page, head, slot)), boxes of 16 rows
// x 64 columns with the 128-byte swizzle.
int make_pool_map(CUtensorMap* map, void* pool, const s3r_kv_cache* c) {
  auto fn = encode_fn();
  if (!fn) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
    return S3R_ERR_CUDA;
  }
  cuuint64_t dims[2] = {(cuuint64_t)c->head_dim,
                        (cuuint64_t)c->num_pages * c->num_kv_heads * S3R_PAGE_SIZE};
  cuuint64_t strides[1] = {(cuuint64_t)c->head_dim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)S3R_PAGE_SIZE};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pool, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled: error %d", (int)r);
    return S3R_ERR_CUDA;
  }
  return S3R_OK;
}

// 4-D view of a pool (d, slot, kv head, page) with boxes of 64 columns x 16 slots x 1 head x
// `pages` pages: `pages` consecutive page ids of one head land as one [pages*16][128 B] block
// (128-byte swizzle), the layout of the 2-D map's 16-row boxes stacked.
int make_paged_map(CUtensorMap* map, void* pool, const s3r_kv_cache* c, int pages) {
  auto fn = encode_fn();
  if (!fn) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
    return S3R_ERR_CUDA;
  }
  const cuuint64_t row = (cuuint64_t)c->head_dim * 2;
  cuuint64_t dims[4] = {(cuuint64_t)c->head_dim, (cuuint64_t)S3R_PAGE_SIZE,
                        (cuuint64_t)c->num_kv_heads, (cuuint64_t)c->num_pages};
  cuuint64_t strides[3] = {row, row * S3R_PAGE_SIZE, row * S3R_PAGE_SIZE * c->num_kv_heads};
  cuuint32_t box[4] = {64, (cuuint32_t)S3R_PAGE_SIZE, 1, (cuuint32_t)pages};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, pool, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (4-D): error %d", (int)r);
    return S3R_ERR_CUDA;
  }
  return S3R_OK;
}

// 3-D view of the query rows q [num_requests][T][H_q][d] as (d, q head, request * T + t)
// with boxes of 64 columns x G heads x T rows: the G*T rows of one (request, KV head) land
// as one [T*G][128 B] block (row t*G + g, 128-byte swizzle) per 64-column half.
int make_q_map(CUtensorMap* map, const void* q, const s3r_kv_cache* c, int num_requests, int T) {
  auto fn = encode_fn();
  if (!fn) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
    return S3R_ERR_CUDA;
  }
  const int G = c->num_q_heads / c->num_kv_heads;
  const cuuint64_t row = (cuuint64_t)c->head_dim * 2;
  cuuint64_t dims[3] = {(cuuint64_t)c->head_dim, (cuuint64_t)c->num_q_heads,
                        (cuuint64_t)num_requests * T};
  cuuint64_t strides[2] = {row, row * c->num_q_heads};
  cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)T};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (q): error %d", (int)r);
    return S3R_ERR_CUDA;
  }
  return S3R_OK;
}

size_t verify_need(const s3r_kv_cache* c, int num_requests, int cap, int k) {
  const int G = c->num_q_heads / c->num_kv_heads;
  return head_bytes(num_requests) +
         verify_partial_bytes(num_requests, c->num_kv_heads, cap, G * (k + 1), c->head_dim,
                              kVerifyChunkMin);
}

size_t draft_need(const s3r_kv_cache* c, int num_requests, int sel_stride) {
  return head_bytes(num_requests) +
         draft_partial_bytes(num_requests, c->num_kv_heads, sel_stride, c->head_dim);
}

size_t sample_need(int num_requests, int hkv, int k, int vocab) {
  return head_bytes(num_requests) + sample_partial_bytes(num_requests, k, vocab);
}

// ---------------------------------------------------- draft sampling without a workspace
// Scratch of s3r_draft_sample_noalloc, a file-scope device array instead of a caller's
// workspace: one arrival ticket per request (cleared by every call for its requests; the
// last block of a request puts it back to zero) followed by one partial record per
// (request, vocabulary chunk) and the eight sub-block sums of each chunk. It is sized for
// S3R_NOALLOC_MAX_REQUESTS requests and vocabularies of at most S3R_NOALLOC_MAX_VOCAB
// entries: 8 KiB of tickets + 1 MiB of partials + 2 MiB of sub-block sums per device.
constexpr int kNoAllocChunks = S3R_NOALLOC_MAX_VOCAB / kVocabChunk;
constexpr size_t kNoAllocTicketBytes = (size_t)S3R_NOALLOC_MAX_REQUESTS * sizeof(int);
constexpr size_t kNoAllocBytes =
    kNoAllocTicketBytes + (size_t)S3R_NOALLOC_MAX_REQUESTS * kNoAllocChunks * kSamplePartialBytes +
    (size_t)S3R_NOALLOC_MAX_REQUESTS * kNoAllocChunks * 8 * sizeof(float);
static_assert(S3R_NOALLOC_MAX_VOCAB % kVocabChunk == 0, "whole vocabulary chunks");
static_assert(kNoAllocTicketBytes % 256 == 0, "partials start 256-byte aligned");

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

namespace {

// Device address of the scratch on the current device. The first call on a device looks
// the symbol up (cudaGetSymbolAddress, no allocation); later calls only read the cached
// address.
int noalloc_scratch(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaGetLastError(), "cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices) return S3R_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    const int st = cuda_status(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress");
    if (st != S3R_OK) return st;
    if ((reinterpret_cast<uintptr_t>(p) & 255u) != 0) return S3R_ERR_WORKSPACE;
    g_noalloc_ptr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_noalloc_ptr[dev]);
  return S3R_OK;
}

#define S3R_TRY(x)              \
  do {                          \
    const int _st = (x);        \
    if (_st != S3R_OK) return _st; \
  } while (0)

}  // namespace

extern "C" {

size_t s3r_workspace_size(const s3r_kv_cache* cache, int32_t num_requests,
                          int32_t max_pages_per_req, int32_t max_k, int32_t vocab,
                          int32_t sel_stride) {
  if (check_cache(cache) != S3R_OK || num_requests < 0 || max_pages_per_req <= 0 || max_k < 0 ||
      max_k > S3R_MAX_K || vocab < 0 || sel_stride < 0)
    return 0;
  const int cap = max_pages_per_req * S3R_PAGE_SIZE;
  size_t need = head_bytes(num_requests);
  size_t a = verify_need(cache, num_requests, cap, max_k);
  size_t b = draft_need(cache, num_requests, sel_stride);
  size_t c = sample_need(num_requests, cache->num_kv_heads, max_k, vocab > 0 ? vocab : 1);
  const size_t d = head_bytes(num_requests) + select_sigma_bytes(num_requests, cache->num_kv_heads, cap);
  if (d > need) need = d;
  if (a > need) need = a;
  if (b > need) need = b;
  if (c > need) need = c;
  return need;
}

int s3r_workspace_init(void* ws, size_t ws_bytes, s3r_stream_t stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < kWsHeader)
    return S3R_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream), "cudaMemsetAsync");
}

int s3r_verify_attn(const s3r_kv_cache* cache, const s3r_batch* batch, int32_t k,
                    const void* q, const void* k_new, const void* v_new, void* out, float* lse,
                    float* score_logits, void* ws, size_t ws_bytes, s3r_stream_t stream) {
  S3R_TRY(check_cache(cache));
  S3R_TRY(check_batch(batch, true));
  if (k < 0 || k > S3R_MAX_K) return S3R_ERR_UNSUPPORTED;
  const int G = cache->num_q_heads / cache->num_kv_heads;
  const int R = G * (k + 1);
  if (R > S3R_MAX_ROWS) return S3R_ERR_UNSUPPORTED;
  if (!q || !k_new || !v_new || !out || !lse) return S3R_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out) ||
      !aligned4(lse) || (score_logits && !aligned16(score_logits)))
    return S3R_ERR_INVALID_ARG;
  if (batch->batch == 0) return S3R_OK;
  const int cap = batch->max_pages_per_req * S3R_PAGE_SIZE;
  S3R_TRY(check_ws(ws, ws_bytes, verify_need(cache, batch->num_requests, cap, k)));
  CUtensorMap tk, tv;
  S3R_TRY(make_pool_map(&tk, cache->k_pool, cache));
  S3R_TRY(make_pool_map(&tv, cache->v_pool, cache));
  const Carve w = carve(ws, batch->num_requests);
  VerifyParams p;
  std::memset(&p, 0, sizeof(p));
  p.req_ids = batch->req_ids;
  p.seq_lens = batch->seq_lens;
  p.num_requests = batch->num_requests;
  p.page_table = batch->page_table;
  p.max_pages = batch->max_pages_per_req;
  p.cap = cap;
  p.Hq = cache->num_q_heads;
  p.Hkv = cache->num_kv_heads;
  p.G = G;
  p.T = k + 1;
  p.R = R;
  p.Rp = ((R + 15) / 16) * 16;
  p.num_pages = cache->num_pages;
  p.k_pool = static_cast<__nv_bfloat16*>(cache->k_pool);
  p.v_pool = static_cast<__nv_bfloat16*>(cache->v_pool);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.scores = score_logits;
  p.scale = 1.0f / sqrtf((float)cache->head_dim);
  p.chunk = kVerifyChunk;
  p.nchunk_max = (cap + kVerifyChunk - 1) / kVerifyChunk;
  p.err = w.err;
  p.tickets = w.tickets;
  p.sched = w.sched;
  p.part = reinterpret_cast<float*>(w.part);
  p.wait_limit = g_wait_limit.load();
  int st;
  const bool tc = g_verify_kernel.load() == 0 && verify_tc_supported(cache->head_dim, R, batch->batch);
  {
    const int chunk = tc ? verify_tc_chunk(R) : kVerifyChunk;
    if (!verify_combine_fits((cap + chunk - 1) / chunk, R)) return S3R_ERR_UNSUPPORTED;
  }
  if (tc) {
    p.Rp = verify_tc_rec_rows(R);
    p.chunk = verify_tc_chunk(R);
    p.nchunk_max = (cap + p.chunk - 1) / p.chunk;
    CUtensorMap k1, v1, k8, v8, qm;
    S3R_TRY(make_q_map(&qm, q, cache, batch->num_requests, k + 1));
    S3R_TRY(make_paged_map(&k1, cache->k_pool, cache, 1));
    S3R_TRY(make_paged_map(&v1, cache->v_pool, cache, 1));
    S3R_TRY(make_paged_map(&k8, cache->k_pool, cache, 8));
    S3R_TRY(make_paged_map(&v8, cache->v_pool, cache, 8));
    int nl = 0;
    st = launch_verify_tc(qm, k1, v1, k8, v8, p, batch->batch, sm_count(), (cudaStream_t)stream, &nl);
    g_launches.fetch_add((uint64_t)nl, std::memory_order_relaxed);
  } else {
    st = launch_verify(tk, tv, p, cache->head_dim, batch->batch, (cudaStream_t)stream);
    if (st == S3R_OK) g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  if (st != S3R_OK) return st;
  return finish(launch_verify_combine(p, cache->head_dim, batch->batch, (cudaStream_t)stream), 1);
}

static int select_common(const s3r_kv_cache* cache, const s3r_batch* batch, SelectParams& p,
                         int32_t budget_bp, int32_t window, int32_t* sel_idx, int32_t sel_stride,
                         int32_t* sel_count, void* ws, size_t ws_bytes, s3r_stream_t stream,
                         int page = 1) {
  if (budget_bp < 1 || budget_bp > 10000 || window < 1) return S3R_ERR_INVALID_ARG;
  if (!sel_idx || !sel_count || sel_stride < 1 || !aligned4(sel_idx) || !aligned4(sel_count))
    return S3R_ERR_INVALID_ARG;
  if (batch->batch > 65535) return S3R_ERR_UNSUPPORTED;   // grid.y
  if (batch->batch == 0) return S3R_OK;
  const size_t need = head_bytes(batch->num_requests) +
                      (p.logits ? select_sigma_bytes(batch->num_requests, cache->num_kv_heads, p.cap) : 0);
  S3R_TRY(check_ws(ws, ws_bytes, need));
  const Carve w = carve(ws, batch->num_requests);
  if (p.logits) p.sigma_buf = reinterpret_cast<float*>(w.part);
  p.req_ids = batch->req_ids;
  p.seq_lens = batch->seq_lens;
  p.Hq = cache->num_q_heads;
  p.Hkv = cache->num_kv_heads;
  p.G = cache->num_q_heads / cache->num_kv_heads;
  p.budget_bp = budget_bp;
  p.window = window;
  p.sel_idx = sel_idx;
  p.sel_stride = sel_stride;
  p.sel_count = sel_count;
  p.err = w.err;
  p.page = page;
  p.num_requests = batch->num_requests;
  p.num_sms = sm_count();
  int nl = 0;
  const int st = launch_select(p, batch->batch, (cudaStream_t)stream, &nl);
  g_launches.fetch_add((uint64_t)nl, std::memory_order_relaxed);
  return st;
}

static int select_kv_impl(const s3r_kv_cache* cache, const s3r_batch* batch,
                          const float* score_logits, const float* lse, int32_t k_prev,
                          int32_t budget_bp, int32_t window, int32_t* sel_idx, int32_t sel_stride,
                          int32_t* sel_count, void* ws, size_t ws_bytes, s3r_stream_t stream,
                          int page) {
  S3R_TRY(check_cache(cache));
  S3R_TRY(check_batch(batch, true));
  if (k_prev < 0 || k_prev > S3R_MAX_K) return S3R_ERR_UNSUPPORTED;
  if (window < k_prev + 1) return S3R_ERR_INVALID_ARG;
  if (!score_logits || !lse || !aligned16(score_logits) || !aligned4(lse))
    return S3R_ERR_INVALID_ARG;
  const int G = cache->num_q_heads / cache->num_kv_heads;
  if (G * (k_prev + 1) > S3R_MAX_ROWS) return S3R_ERR_UNSUPPORTED;
  SelectParams p;
  std::memset(&p, 0, sizeof(p));
  p.cap = batch->max_pages_per_req * S3R_PAGE_SIZE;
  p.logits = score_logits;
  p.lse = lse;
  p.T = k_prev + 1;
  p.R = G * (k_prev + 1);
  return select_common(cache, batch, p, budget_bp, window, sel_idx, sel_stride, sel_count, ws,
                       ws_bytes, stream, page);
}

static int select_from_scores_impl(const s3r_kv_cache* cache, const s3r_batch* batch,
                                   const float* scores, int32_t score_stride, int32_t budget_bp,
                                   int32_t window, int32_t* sel_idx, int32_t sel_stride,
                                   int32_t* sel_count, void* ws, size_t ws_bytes,
                                   s3r_stream_t stream, int page) {
  S3R_TRY(check_cache(cache));
  S3R_TRY(check_batch(batch, false));
  if (!scores || !aligned4(scores) || score_stride < 1) return S3R_ERR_INVALID_ARG;
  SelectParams p;
  std::memset(&p, 0, sizeof(p));
  p.scores = scores;
  p.score_stride = score_stride;
  return select_common(cache, batch, p, budget_bp, window, sel_idx, sel_stride, sel_count, ws,
                       ws_bytes, stream, page);
}

int s3r_select_kv(const s3r_kv_cache* cache, const s3r_batch* batch, const float* score_logits,
                  const float* lse, int32_t k_prev, int32_t budget_bp, int32_t window,
                  int32_t* sel_idx, int32_t sel_stride, int32_t* sel_count, void* ws,
                  size_t ws_bytes, s3r_stream_t stream) {
  return select_kv_impl(cache, batch, score_logits, lse, k_prev, budget_bp, window, sel_idx,
                        sel_stride, sel_count, ws, ws_bytes, stream, 1);
}

int s3r_select_kv_pages(const s3r_kv_cache* cache, const s3r_batch* batch,
                        const float* score_logits, const float* lse, int32_t k_prev,
                        int32_t budget_bp, int32_t window, int32_t* sel_idx, int32_t sel_stride,
                        int32_t* sel_count, void* ws, size_t ws_bytes, s3r_stream_t stream) {
  return select_kv_impl(cache, batch, score_logits, lse, k_prev, budget_bp, window, sel_idx,
                        sel_stride, sel_count, ws, ws_bytes, stream, S3R_PAGE_SIZE);
}

int s3r_position_scores(const s3r_kv_cache* cache, const s3r_batch* batch,
                        const float* score_logits, const float* lse, int32_t k_prev,
                        float* scores, int32_t score_stride, void* ws, size_t ws_bytes,
                        s3r_stream_t stream) {
  S3R_TRY(check_cache(cache));
  S3R_TRY(check_batch(batch, true));
  if (k_prev < 0 || k_prev > S3R_MAX_K) return S3R_ERR_UNSUPPORTED;
  const int G = cache->num_q_heads / cache->num_kv_heads;
  if (G * (k_prev + 1) > S3R_MAX_ROWS) return S3R_ERR_UNSUPPORTED;
  if (!score_logits || !lse || !scores || !aligned16(score_logits) || !aligned4(lse) ||
      !aligned16(scores) || score_stride < 1 || (score_stride % 4))
    return S3R_ERR_INVALID_ARG;
  if (batch->batch > 65535) return S3R_ERR_UNSUPPORTED;   // grid.z
  if (batch->batch == 0) return S3R_OK;
  S3R_TRY(check_ws(ws, ws_bytes, head_bytes(batch->num_requests)));
  const Carve w = carve(ws, batch->num_requests);
  SelectParams p;
  std::memset(&p, 0, sizeof(p));
  p.req_ids = batch->req_ids;
  p.seq_lens = batch->seq_lens;
  p.Hq = cache->num_q_heads;
  p.Hkv = cache->num_kv_heads;
  p.G = G;
  p.cap = batch->max_pages_per_req * S3R_PAGE_SIZE;
  p.logits = score_logits;
  p.lse = lse;
  p.T = k_prev + 1;
  p.R = G * (k_prev + 1);
  p.window = 0;   // every committed position
  p.sigma_buf = scores;
  p.sigma_stride = score_stride;
  p.err = w.err;
  p.num_requests = batch->num_requests;
  const int st = launch_sigma(p, batch->batch, (cudaStream_t)stream);
  if (st == S3R_OK) g_launches.fetch_add(1, std::memory_order_relaxed);
  return st;
}

int s3r_select_from_scores(const s3r_kv_cache* cache, const s3r_batch* batch,
                           const float* scores, int32_t score_stride, int32_t budget_bp,
                           int32_t window, int32_t* sel_idx, int32_t sel_stride,
                           int32_t* sel_count, void* ws, size_t ws_bytes, s3r_stream_t stream) {
  return select_from_scores_impl(cache, batch, scores, score_stride, budget_bp, window, sel_idx,
                                 sel_stride, sel_count, ws, ws_bytes, stream, 1);
}

int s3r_select_pages_from_scores(const s3r_kv_cache* cache, const s3r_batch* batch,
                                 const float* scores, int32_t score_stride, int32_t budget_bp,
                                 int32_t window, int32_t* sel_idx, int32_t sel_stride,
                                 int32_t* sel_count, void* ws, size_t ws_bytes,
                                 s3r_stream_t stream) {
  return select_from_scores_impl(cache, batch, scores, score_stride, budget_bp, window, sel_idx,
                                 sel_stride, sel_count, ws, ws_bytes, stream, S3R_PAGE_SIZE);
}

int s3r_sparse_draft_attn(const s3r_kv_cache* cache, const s3r_batch* batch,
                          const int32_t* draft_step, const void* q, int32_t q_stride,
                          const void* k_new, const void* v_new, int32_t kv_stride,
                          const int32_t* sel_idx, int32_t sel_stride,
                          const int32_t* sel_count, void* out, float* lse, void* ws,
                          size_t ws_bytes, s3r_stream_t stream) {
  S3R_TRY(check_cache(cache));
  S3R_TRY(check_batch(batch, true));
  if (!draft_step || !q || !k_new || !v_new || !sel_idx || !sel_count || !out)
    return S3R_ERR_INVALID_ARG;
  if (!aligned4(draft_step) || !aligned16(q) || !aligned16(k_new) || !aligned16(v_new) ||
      !aligned4(sel_idx) || !aligned4(sel_count) || !aligned16(out) || (lse && !aligned4(lse)))
    return S3R_ERR_INVALID_ARG;
  if (sel_stride < 1) return S3R_ERR_INVALID_ARG;
  const int64_t qrow = (int64_t)cache->num_q_heads * cache->head_dim;
  const int64_t kvrow = (int64_t)cache->num_kv_heads * cache->head_dim;
  if (q_stride == 0) q_stride = (int32_t)qrow;
  if (kv_stride == 0) kv_stride = (int32_t)kvrow;
  if (q_stride < qrow || kv_stride < kvrow || (q_stride % 8) || (kv_stride % 8))
    return S3R_ERR_INVALID_ARG;
  if (batch->batch == 0) return S3R_OK;
  S3R_TRY(check_ws(ws, ws_bytes, draft_need(cache, batch->num_requests, sel_stride)));
  const Carve w = carve(ws, batch->num_requests);
  DraftParams p;
  std::memset(&p, 0, sizeof(p));
  p.req_ids = batch->req_ids;
  p.seq_lens = batch->seq_lens;
  p.page_table = batch->page_table;
  p.max_pages = batch->max_pages_per_req;
  p.cap = batch->max_pages_per_req * S3R_PAGE_SIZE;
  p.Hq = cache->num_q_heads;
  p.Hkv = cache->num_kv_heads;
  p.G = cache->num_q_heads / cache->num_kv_heads;
  p.num_pages = cache->num_pages;
  p.k_pool = static_cast<__nv_bfloat16*>(cache->k_pool);
  p.v_pool = static_cast<__nv_bfloat16*>(cache->v_pool);
  p.draft_step = draft_step;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.q_stride = q_stride;
  p.kv_stride = kv_stride;
  p.sel_idx = sel_idx;
  p.sel_stride = sel_stride;
  p.sel_count = sel_count;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.scale = 1.0f / sqrtf((float)cache->head_dim);
  p.err = w.err;
  p.tickets = w.tickets;
  p.part = reinterpret_cast<float*>(w.part);
  p.nchunk_max = (sel_stride + S3R_MAX_K + 1 + kDraftChunk - 1) / kDraftChunk;
  p.num_requests = batch->num_requests;
  int nl = 0;
  const int st = launch_draft(p, cache->head_dim, batch->batch, sm_count(), (cudaStream_t)stream, &nl);
  g_launches.fetch_add((uint64_t)nl, std::memory_order_relaxed);
  return st;
}

int s3r_draft_sample(const s3r_batch* batch, const int32_t* draft_step, int32_t k,
                     const float* q_logits, int32_t vocab, uint64_t seed, int32_t* draft_tokens,
                     float* margins, s3r_row_norm* q_norm, void* ws, size_t ws_bytes,
                     s3r_stream_t stream) {
  S3R_TRY(check_batch(batch, false));
  if (k < 1 || k > S3R_MAX_K) return S3R_ERR_UNSUPPORTED;
  if (vocab < 1 || vocab > 64 * kVocabChunk) return S3R_ERR_UNSUPPORTED;
  if (!draft_step || !q_logits || !draft_tokens || !aligned4(draft_step) ||
      !aligned4(q_logits) || !aligned4(draft_tokens) || (margins && !aligned4(margins)) ||
      (q_norm && (reinterpret_cast<uintptr_t>(q_norm) & 7u)))
    return S3R_ERR_INVALID_ARG;
  if (batch->batch == 0) return S3R_OK;
  S3R_TRY(check_ws(ws, ws_bytes, sample_need(batch->num_requests, 1, k, vocab)));
  const Carve w = carve(ws, batch->num_requests);
  SampleParams p;
  std::memset(&p, 0, sizeof(p));
  p.req_ids = batch->req_ids;
  p.seq_lens = batch->seq_lens;
  p.draft_step = draft_step;
  p.k = k;
  p.vocab = vocab;
  p.nvch = nvch_of(vocab);
  p.q_logits = q_logits;
  p.draft_out = draft_tokens;
  p.seed = seed;
  p.err = w.err;
  p.tickets = w.tickets;
  p.part = w.part;
  p.num_requests = batch->num_requests;
  p.margins = margins;
  p.q_norm = q_norm;
  p.sub_off = draft_sub_offset(batch->num_requests, vocab);
  return finish(launch_draft_sample(p, batch->batch, (cudaStream_t)stream), 1);
}

int s3r_draft_sample_noalloc(const s3r_batch* batch, const int32_t* draft_step, int32_t k,
                             const float* q_logits, int32_t vocab, uint64_t seed,
                             int32_t* draft_tokens, int32_t* err_word, s3r_stream_t stream) {
  g_last_error[0] = '\0';
  S3R_TRY(check_batch(batch, false));
  if (k < 1 || k > S3R_MAX_K) return S3R_ERR_UNSUPPORTED;
  if (vocab < 1) return S3R_ERR_UNSUPPORTED;
  if (!draft_step || !q_logits || !draft_tokens || !err_word || !aligned4(draft_step) ||
      !aligned4(q_logits) || !aligned4(draft_tokens) || !aligned4(err_word))
    return S3R_ERR_INVALID_ARG;
  if (batch->num_requests > S3R_NOALLOC_MAX_REQUESTS || vocab > S3R_NOALLOC_MAX_VOCAB) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "s3r_draft_sample_noalloc: %d requests / vocab %d exceed the static scratch "
                  "(at most %d requests, vocab %d)",
                  batch->num_requests, vocab, S3R_NOALLOC_MAX_REQUESTS, S3R_NOALLOC_MAX_VOCAB);
    return S3R_ERR_UNSUPPORTED;
  }
  if (batch->batch == 0) return S3R_OK;
  unsigned char* scratch = nullptr;
  S3R_TRY(noalloc_scratch(&scratch));
  SampleParams p;
  std::memset(&p, 0, sizeof(p));
  p.req_ids = batch->req_ids;
  p.seq_lens = batch->seq_lens;
  p.draft_step = draft_step;
  p.k = k;
  p.vocab = vocab;
  p.nvch = nvch_of(vocab);
  p.q_logits = q_logits;
  p.draft_out = draft_tokens;
  p.seed = seed;
  p.err = err_word;
  p.tickets = reinterpret_cast<int*>(scratch);
  p.part = scratch + kNoAllocTicketBytes;
  p.num_requests = batch->num_requests;
  p.sub_off = draft_sub_offset(batch->num_requests, vocab);
  // the tickets of this call's requests start at zero whatever an earlier call left there,
  // cleared on the call's own stream (so ordered with the launch below)
  S3R_TRY(cuda_status(cudaMemsetAsync(scratch, 0, (size_t)batch->num_requests * sizeof(int),
                                      (cudaStream_t)stream), "cudaMemsetAsync"));
  return finish(launch_draft_sample(p, batch->batch, (cudaStream_t)stream), 1);
}

int s3r_spec_sample(const s3r_batch* batch, int32_t k, const float* p_logits,
                    const float* q_logits, const int32_t* draft_tokens, int32_t vocab,
                    uint64_t seed, int32_t* out_tokens, int32_t* n_out, float* margins,
                    const s3r_row_norm* q_norm, void* ws, size_t ws_bytes, s3r_stream_t stream) {
  S3R_TRY(check_batch(batch, false));
  if (k < 0 || k > S3R_MAX_K) return S3R_ERR_UNSUPPORTED;
  if (vocab < 1 || vocab > 64 * kVocabChunk) return S3R_ERR_UNSUPPORTED;
  if (!p_logits || !out_tokens || !n_out || !aligned4(p_logits) || !aligned4(out_tokens) ||
      !aligned4(n_out) || (margins && !aligned4(margins)) ||
      (q_norm && (reinterpret_cast<uintptr_t>(q_norm) & 7u)))
    return S3R_ERR_INVALID_ARG;
  if (k > 0 && (!q_logits || !draft_tokens || !aligned4(q_logits) || !aligned4(draft_tokens)))
    return S3R_ERR_INVALID_ARG;
  if (batch->batch == 0) return S3R_OK;
  S3R_TRY(check_ws(ws, ws_bytes, sample_need(batch->num_requests, 1, k, vocab)));
  const Carve w = carve(ws, batch->num_requests);
  SampleParams p;
  std::memset(&p, 0, sizeof(p));
  p.req_ids = batch->req_ids;
  p.seq_lens = batch->seq_lens;
  p.k = k;
  p.vocab = vocab;
  p.nvch = nvch_of(vocab);
  p.p_logits = p_logits;
  p.q_logits = q_logits;
  p.draft_tokens = draft_tokens;
  p.out_tokens = out_tokens;
  p.n_out = n_out;
  p.seed = seed;
  p.err = w.err;
  p.tickets = w.tickets;
  p.part = w.part;
  p.num_requests = batch->num_requests;
  p.margins = margins;
  p.q_norm = const_cast<s3r_row_norm*>(q_norm);
  spec_offsets(batch->num_requests, k, vocab, &p.plan_off, &p.draw_off, &p.sub_off);
  int launches = 0;
  const int st = launch_spec_sample(p, batch->batch, (cudaStream_t)stream, &launches);
  if (st != S3R_OK && launches == 0) return st;
  g_launches.fetch_add((uint64_t)(st == S3R_OK ? launches : 1), std::memory_order_relaxed);
  return st;
}

int s3r_draft_argmax(const s3r_batch* batch, const int32_t* draft_step, int32_t k,
                     const float* q_logits, int32_t vocab, int32_t* draft_tokens, void* ws,
                     size_t ws_bytes, s3r_stream_t stream) {
  S3R_TRY(check_batch(batch, false));
  if (k < 1 || k > S3R_MAX_K) return S3R_ERR_UNSUPPORTED;
  if (vocab < 1 || vocab > 64 * kVocabChunk) return S3R_ERR_UNSUPPORTED;
  if (!draft_step || !q_logits || !draft_tokens || !aligned4(draft_step) ||
      !aligned4(q_logits) || !aligned4(draft_tokens))
    return S3R_ERR_INVALID_ARG;
  if (batch->batch == 0) return S3R_OK;
  S3R_TRY(check_ws(ws, ws_bytes, sample_need(batch->num_requests, 1, k, vocab)));
  const Carve w = carve(ws, batch->num_requests);
  SampleParams p;
  std::memset(&p, 0, sizeof(p));
  p.req_ids = batch->req_ids;
  p.seq_lens = batch->seq_lens;
  p.draft_step = draft_step;
  p.k = k;
  p.vocab = vocab;
  p.nvch = nvch_of(vocab);
  p.q_logits = q_logits;
  p.draft_out = draft_tokens;
  p.err = w.err;
  p.tickets = w.tickets;
  p.part = w.part;
  p.num_requests = batch->num_requests;
  return finish(launch_argmax(p, batch->batch, 0, (cudaStream_t)stream), 1);
}

int s3r_greedy_verify(const s3r_batch* batch, int32_t k, const float* p_logits,
                      const int32_t* draft_tokens, int32_t vocab, int32_t* out_tokens,
                      int32_t* n_out, void* ws, size_t ws_bytes, s3r_stream_t stream) {
  S3R_TRY(check_batch(batch, false));
  if (k < 0 || k > S3R_MAX_K) return S3R_ERR_UNSUPPORTED;
  if (vocab < 1 || vocab > 64 * kVocabChunk) return S3R_ERR_UNSUPPORTED;
  if (!p_logits || !out_tokens || !n_out || !aligned4(p_logits) || !aligned4(out_tokens) ||
      !aligned4(n_out))
    return S3R_ERR_INVALID_ARG;
  if (k > 0 && (!draft_tokens || !aligned4(draft_tokens))) return S3R_ERR_INVALID_ARG;
  if (batch->batch == 0) return S3R_OK;
  S3R_TRY(check_ws(ws, ws_bytes, sample_need(batch->num_requests, 1, k, vocab)));
  const Carve w = carve(ws, batch->num_requests);
  SampleParams p;
  std::memset(&p, 0, sizeof(p));
  p.req_ids = batch->req_ids;
  p.seq_lens = batch->seq_lens;
  p.k = k;
  p.vocab = vocab;
  p.nvch = nvch_of(vocab);
  p.p_logits = p_logits;
  p.draft_tokens = draft_tokens;
  p.out_tokens = out_tokens;
  p.n_out = n_out;
  p.err = w.err;
  p.tickets = w.tickets;
  p.part = w.part;
  p.num_requests = batch->num_requests;
  return finish(launch_argmax(p, batch->batch, 1, (cudaStream_t)stream), 1);
}

int s3r_commit(const s3r_batch* batch, int32_t k, const int32_t* n_out, int32_t* seq_lens,
               int64_t* stats, s3r_stream_t stream) {
  S3R_TRY(check_batch(batch, false));
  if (k < 0 || k > S3R_MAX_K) return S3R_ERR_UNSUPPORTED;
  if (!n_out || !seq_lens || !aligned4(n_out) || !aligned4(seq_lens)) return S3R_ERR_INVALID_ARG;
  if (stats && (reinterpret_cast<uintptr_t>(stats) & 7u)) return S3R_ERR_INVALID_ARG;
  if (batch->batch == 0) return S3R_OK;
  return finish(launch_commit(batch->req_ids, batch->batch, batch->num_requests, k, n_out, seq_lens, stats,
                              (cudaStream_t)stream),
                1);
}

// Smoothed acceptance per position (the reading of s3r_choose_horizon), or false for an
// argument it rejects.
static bool horizon_alpha(const double* accepted, const double* decided, int32_t k_max, double prior_alpha,
                          double prior_weight, double* alpha) {
  if (!(prior_alpha >= 0.0 && prior_alpha <= 1.0) || !(prior_weight >= 0.0) || !std::isfinite(prior_weight))
    return false;
  for (int j = 0; j < k_max; ++j) {
    if (!(accepted[j] >= 0.0) || !(decided[j] >= 0.0) || !std::isfinite(accepted[j]) ||
        !std::isfinite(decided[j]) || decided[j] + prior_weight == 0.0)
      return false;
    alpha[j] = (accepted[j] + prior_weight * prior_alpha) / (decided[j] + prior_weight);
  }
  return true;
}

// The k in [1, k_max] with the most expected tokens per unit cost, cost[k-1] the round's
// cost at length k; the smallest k on ties.
static int horizon_pick(const double* alpha, int32_t k_max, const double* cost) {
  int best_k = 1;
  double best = -1.0, tau = 1.0, run = 1.0;
  for (int k = 1; k <= k_max; ++k) {
    run *= alpha[k - 1];
    tau += run;
    const double rate = tau / cost[k - 1];
    if (rate > best) {
      best = rate;
      best_k = k;
    }
  }
  return best_k;
}

static bool costs_ok(const double* round_cost, int32_t k_max) {
  for (int k = 0; k < k_max; ++k)
    if (!(round_cost[k] > 0.0) || !std::isfinite(round_cost[k])) return false;
  return true;
}

int s3r_choose_horizon(const double* accepted, const double* decided, int32_t k_max,
                       double c_draft, double c_verify, double prior_alpha, double prior_weight,
                       int32_t* k_out) {
  if (!accepted || !decided || !k_out || k_max < 1 || k_max > S3R_MAX_K) return S3R_ERR_INVALID_ARG;
  if (!(c_draft > 0.0) || !(c_verify > 0.0) || !std::isfinite(c_draft) || !std::isfinite(c_verify))
    return S3R_ERR_INVALID_ARG;
  double alpha[S3R_MAX_K];
  if (!horizon_alpha(accepted, decided, k_max, prior_alpha, prior_weight, alpha)) return S3R_ERR_INVALID_ARG;
  double cost[S3R_MAX_K];
  for (int k = 1; k <= k_max; ++k) cost[k - 1] = (double)k * c_draft + c_verify;
  *k_out = horizon_pick(alpha, k_max, cost);
  return S3R_OK;
}

int s3r_choose_horizon_costs(const double* accepted, const double* decided, int32_t k_max,
                             const double* round_cost, double prior_alpha, double prior_weight,
                             int32_t* k_out) {
  if (!accepted || !decided || !round_cost || !k_out || k_max < 1 || k_max > S3R_MAX_K)
    return S3R_ERR_INVALID_ARG;
  if (!costs_ok(round_cost, k_max)) return S3R_ERR_INVALID_ARG;
  double alpha[S3R_MAX_K];
  if (!horizon_alpha(accepted, decided, k_max, prior_alpha, prior_weight, alpha)) return S3R_ERR_INVALID_ARG;
  *k_out = horizon_pick(alpha, k_max, round_cost);
  return S3R_OK;
}

// The counter update of s3r_horizon_step into acc / dec / *prior (the caller's arrays are
// not touched yet); false for an argument it rejects.
static bool horizon_counts(const int64_t* stats_now, const int64_t* stats_last, const double* accepted,
                           const double* decided, int32_t k_max, double decay, double prior_alpha, double* acc,
                           double* dec, double* prior) {
  if (k_max < 1 || k_max > S3R_MAX_K || !(decay >= 0.0 && decay <= 1.0)) return false;
  for (int j = 0; j < S3R_MAX_K; ++j) {
    const int64_t da = stats_now[2 + j] - stats_last[2 + j];
    const int64_t dd = stats_now[2 + S3R_MAX_K + j] - stats_last[2 + S3R_MAX_K + j];
    if (da < 0 || dd < 0) return false;
    acc[j] = decay * accepted[j] + (double)da;
    dec[j] = decay * decided[j] + (double)dd;
  }
  *prior = prior_alpha;
  if (prior_alpha < 0.0) {
    double sa = 0.0, sd = 0.0;
    for (int j = 0; j < k_max; ++j) {
      sa += acc[j];
      sd += dec[j];
    }
    *prior = sd > 0.0 ? sa / sd : 0.5;
  }
  return true;
}

// Commit a horizon step: the decayed counts, the counters seen, the prior and the length.
static void horizon_commit(const int64_t* stats_now, int64_t* stats_last, double* accepted, double* decided,
                           const double* acc, const double* dec, double prior, int32_t k, double* prior_out,
                           int32_t* k_out) {
  for (int j = 0; j < S3R_MAX_K; ++j) {
    accepted[j] = acc[j];
    decided[j] = dec[j];
  }
  for (int j = 0; j < 2 + 2 * S3R_MAX_K; ++j) stats_last[j] = stats_now[j];
  if (prior_out) *prior_out = prior;
  *k_out = k;
}

int s3r_horizon_step(const int64_t* stats_now, int64_t* stats_last, double* accepted,
                     double* decided, int32_t k_max, double decay, double c_draft,
                     double c_verify, double prior_alpha, double prior_weight,
                     double* prior_out, int32_t* k_out) {
  if (!stats_now || !stats_last || !accepted || !decided || !k_out) return S3R_ERR_INVALID_ARG;
  double acc[S3R_MAX_K], dec[S3R_MAX_K], prior = 0.0;
  if (!horizon_counts(stats_now, stats_last, accepted, decided, k_max, decay, prior_alpha, acc, dec, &prior))
    return S3R_ERR_INVALID_ARG;
  int32_t k = 0;
  const int st = s3r_choose_horizon(acc, dec, k_max, c_draft, c_verify, prior, prior_weight, &k);
  if (st != S3R_OK) return st;
  horizon_commit(stats_now, stats_last, accepted, decided, acc, dec, prior, k, prior_out, k_out);
  return S3R_OK;
}

int s3r_horizon_step_costs(const int64_t* stats_now, int64_t* stats_last, double* accepted,
                           double* decided, int32_t k_max, double decay, const double* round_cost,
                           double prior_alpha, double prior_weight, double* prior_out, int32_t* k_out) {
  if (!stats_now || !stats_last || !accepted || !decided || !k_out) return S3R_ERR_INVALID_ARG;
  double acc[S3R_MAX_K], dec[S3R_MAX_K], prior = 0.0;
  if (!horizon_counts(stats_now, stats_last, accepted, decided, k_max, decay, prior_alpha, acc, dec, &prior))
    return S3R_ERR_INVALID_ARG;
  int32_t k = 0;
  const int st = s3r_choose_horizon_costs(acc, dec, k_max, round_cost, prior, prior_weight, &k);
  if (st != S3R_OK) return st;
  horizon_commit(stats_now, stats_last, accepted, decided, acc, dec, prior, k, prior_out, k_out);
  return S3R_OK;
}

int s3r_philox(uint64_t seed, int32_t stream_id, const int32_t* request, const int32_t* position,
               int64_t n, uint32_t* words, float* u, s3r_stream_t stream) {
  if (n < 0 || (n > 0 && (!request || !position))) return S3R_ERR_INVALID_ARG;
  if (n == 0) return S3R_OK;
  if (n > ((int64_t)1 << 31) * 255) return S3R_ERR_UNSUPPORTED;
  return finish(launch_philox(seed, stream_id, request, position, n, words, u,
                              (cudaStream_t)stream),
                1);
}

int s3r_get_error(void* ws, int32_t* device_error, s3r_stream_t stream) {
  if (!ws || !device_error) return S3R_ERR_INVALID_ARG;
  int32_t v = 0;
  const cudaStream_t st = (cudaStream_t)stream;
  S3R_TRY(cuda_status(cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st), "cudaMemcpyAsync"));
  S3R_TRY(cuda_status(cudaStreamSynchronize(st), "cudaStreamSynchronize"));
  *device_error = v;
  if (v) S3R_TRY(cuda_status(cudaMemsetAsync(ws, 0, sizeof(v), st), "cudaMemsetAsync"));
  S3R_TRY(cuda_status(cudaStreamSynchronize(st), "cudaStreamSynchronize"));
  return S3R_OK;
}

const char* s3r_status_string(int status) {
  switch (status) {
    case S3R_OK: return "ok";
    case S3R_ERR_INVALID_ARG: return "invalid argument";
    case S3R_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case S3R_ERR_CUDA: return "CUDA runtime error";
    case S3R_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case S3R_ERR_DEVICE_BOUNDS: return "device: index, page id or length out of range";
    case S3R_ERR_NONFINITE: return "device: non-finite logit or score";
    case S3R_ERR_TIMEOUT: return "device: bounded wait expired";
    default: return "unknown status";
  }
}

uint64_t s3r_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* s3r_last_error_message(void) { return g_last_error; }

int s3r_set_verify_kernel(int32_t which) {
  if (which < 0 || which > 1) return S3R_ERR_INVALID_ARG;
  g_verify_kernel.store(which);
  return S3R_OK;
}

int s3r_set_wait_limit(int32_t polls) {
  if (polls < 0) return S3R_ERR_INVALID_ARG;
  g_wait_limit.store(polls == 0 ? kWaitLimit : polls);
  return S3R_OK;
}

}  // extern "C"
