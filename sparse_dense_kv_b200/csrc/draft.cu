// Sparse self-draft attention.
//
// What it computes ([News] Interpretation; [Explainer] "How is this different": the draft
// reads a sparse subset of the same KV cache with the same weights): draft step i of
// request r (token at position L+i) writes that token's K/V into its page and lets the G
// query rows of each KV head attend A_i = S ∪ {L, .., L+i}, S the selected positions.
//
// Layout of the work: grid (kv_head, request, chunk of A_i), 128 threads: the block
// scheduler starts every pair's first chunk before any second chunk, so the CTAs that spill
// past the resident ones are mostly the short last chunks of the largest pairs. Chunks are
// kDraftChunk (512) positions long, except that the last one also takes a remainder of up to
// kDraftFold positions instead of leaving it to a CTA of its own. The CTA first resolves the
// element offsets of its positions (selected index, loaded with the set size -> page ->
// slot), then gathers 256-byte K and V rows with 16-byte cp.async (16 lanes per row,
// coalesced) into a 2-stage pipeline laid out like the TMA tiles of the verify (128-byte
// swizzle), so the same tensor-core step (one n-tile of 8 rows per warp) serves both.
// Chunks merge through the workspace in the last CTA of the (request, head), up to four
// records in one round trip; a set that fits one chunk is normalised by its CTA directly,
// with no record and no ticket.
#include "attention.cuh"
#include "kernels.h"

namespace s3r {

constexpr int kDraftStages = 2;
constexpr int kDraftFold = 128;
constexpr int kDraftSpan = kDraftChunk + kDraftFold;   // longest chunk

// Chunks of a set of A positions: ceil(A / kDraftChunk), less one when the last would hold
// at most kDraftFold positions (that remainder goes to the chunk before it).
__device__ __forceinline__ int draft_nchunks(int A) {
  return max(1, (A + kDraftChunk - 1 - kDraftFold) / kDraftChunk);
}

// Merge weights of the 4 position-slice warps of each of the G rows, once per (slice, row):
// fw[s][row] = 2^(m_s - M) (0 for an empty slice), M the rows' maximum, L = sum_s fw l_s
// (in slice order). Ends with a barrier.
template <int RW>
__device__ __forceinline__ void slice_weights(const float* redM, const float* redL, int G, float* fw,
                                              float* Mrow, float* Lrow, int tid) {
  if (tid < G) {
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < 4; ++s) M = fmaxf(M, redM[s * RW + tid]);
    float lsum = 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const float ms = redM[s * RW + tid];
      const float f = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
      fw[s * RW + tid] = f;
      lsum += f * redL[s * RW + tid];
    }
    Mrow[tid] = M;
    Lrow[tid] = lsum;
  }
  __syncthreads();
}

// One chunk's record [m: RW][l: RW][O: RW][D] from the slices (rows below G).
template <int D, int RW>
__device__ __forceinline__ void slices_to_record(const float* redO, const float* fw, const float* Mrow,
                                                 const float* Lrow, int G, float* rec, int tid, int nthreads) {
  constexpr int DS = D + 4;
  for (int v = tid; v < G * (D / 4); v += nthreads) {
    const int row = v / (D / 4), d0 = 4 * (v - row * (D / 4));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const float f = fw[s * RW + row];
      const float4 o = *reinterpret_cast<const float4*>(redO + ((size_t)s * RW + row) * DS + d0);
      acc.x += f * o.x;
      acc.y += f * o.y;
      acc.z += f * o.z;
      acc.w += f * o.w;
    }
    *reinterpret_cast<float4*>(rec + 2 * RW + (size_t)row * D + d0) = acc;
    if (d0 == 0) {
      rec[row] = Mrow[row];
      rec[RW + row] = Lrow[row];
    }
  }
}

// The G rows of a set held by one CTA: normalised outputs and LSE straight from the slices,
// with the operations (and their order) of a one-record merge followed by the combine of
// that single record.
template <int D, int RW, class OutPtr, class LsePtr>
__device__ __forceinline__ void slices_to_output(const float* redO, const float* fw, const float* Mrow,
                                                 const float* Lrow, int G, OutPtr out_row, LsePtr lse_row,
                                                 int tid, int nthreads) {
  constexpr int DS = D + 4;
  for (int v = tid; v < G * (D / 4); v += nthreads) {
    const int row = v / (D / 4), d0 = 4 * (v - row * (D / 4));
    const float M = Mrow[row], lsum = Lrow[row];
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const float f = fw[s * RW + row];
      const float4 o = *reinterpret_cast<const float4*>(redO + ((size_t)s * RW + row) * DS + d0);
      acc[0] += f * o.x;
      acc[1] += f * o.y;
      acc[2] += f * o.z;
      acc[3] += f * o.w;
    }
    const float w = (M == -INFINITY) ? 0.f : exp2f(M - M) / lsum;
    float a[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      a[e] = 0.f;
      a[e] += w * acc[e];
    }
    __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(out_row(row) + d0);
    o[0] = __floats2bfloat162_rn(a[0], a[1]);
    o[1] = __floats2bfloat162_rn(a[2], a[3]);
    if (d0 == 0) {
      float* lp = lse_row(row);
      if (lp) *lp = (M + log2f(lsum)) * kLn2;
    }
  }
}

// The combine of up to kDraftFastMerge chunk records, each thread for 4 consecutive d of one
// row: the records' maxima, sums and O values are all loaded before any is used (one round
// trip), then the combine's operations in its order (row maximum, sum of the weighted
// sums, weights 2^(m_c - M) / sum, weighted sum of O over the chunks).
constexpr int kDraftFastMerge = 4;
template <int D, int RW, class OutPtr, class LsePtr>
__device__ __forceinline__ void combine_few_records(const float* recs, size_t rec_floats, int nch, int G,
                                                    OutPtr out_row, LsePtr lse_row, int tid, int nthreads) {
  for (int v = tid; v < G * (D / 4); v += nthreads) {
    const int row = v / (D / 4), d4 = v - row * (D / 4);
    float mc[kDraftFastMerge], lc[kDraftFastMerge];
    float4 x[kDraftFastMerge];
#pragma unroll
    for (int c = 0; c < kDraftFastMerge; ++c) {
      if (c < nch) {
        const float* rc = recs + c * rec_floats;
        mc[c] = __ldcg(rc + row);
        lc[c] = __ldcg(rc + RW + row);
        x[c] = __ldcg(reinterpret_cast<const float4*>(rc + 2 * RW + (size_t)row * D) + d4);
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kDraftFastMerge; ++c)
      if (c < nch) M = fmaxf(M, mc[c]);
    float lsum = 0.f;
#pragma unroll
    for (int c = 0; c < kDraftFastMerge; ++c)
      if (c < nch) lsum += (mc[c] == -INFINITY) ? 0.f : exp2f(mc[c] - M) * lc[c];
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < kDraftFastMerge; ++c) {
      if (c < nch) {
        const float w = (mc[c] == -INFINITY) ? 0.f : exp2f(mc[c] - M) / lsum;
        a.x += w * x[c].x;
        a.y += w * x[c].y;
        a.z += w * x[c].z;
        a.w += w * x[c].w;
      }
    }
    __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(out_row(row) + 4 * d4);
    o[0] = __floats2bfloat162_rn(a.x, a.y);
    o[1] = __floats2bfloat162_rn(a.z, a.w);
    if (d4 == 0) {
      float* lp = lse_row(row);
      if (lp) *lp = (M + log2f(lsum)) * kLn2;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128) draft_kernel(const DraftParams p) {
  pdl_wait();
  static_assert(kDraftChunk % 128 == 0 && kDraftSpan % 128 == 0, "128 threads resolve the chunk's rows");
  constexpr int NTW = 1, RW = 8, STAGE = 2 * kTile * D * 2, CPR = D / 8;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                             ~uintptr_t(1023));
  int64_t* rowoff = reinterpret_cast<int64_t*>(smem + kDraftStages * STAGE);
  __shared__ int s_flag_mem;
  int* s_flag = &s_flag_mem;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kvh = blockIdx.x, bl = blockIdx.y, c = blockIdx.z;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) {
    if (c == 0 && kvh == 0 && tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int Hkv = p.Hkv, G = p.G;
  // The chunk's selected indices are loaded before the set size is known (within the set's
  // row of sel_stride entries; those past the size are not used), so these loads and the
  // length / step / size loads make one round trip.
  constexpr int kPer = kDraftSpan / 128;
  const int* sel = p.sel_idx + ((size_t)r * Hkv + kvh) * p.sel_stride;
  int selv[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int a = c * kDraftChunk + tid + 128 * u;
    selv[u] = a < p.sel_stride ? __ldg(sel + a) : -1;
  }
  const int L = p.seq_lens[r];
  const int i = p.draft_step[r];
  const int n = p.sel_count[(size_t)r * Hkv + kvh];
  if (L < 0 || i < 0 || i >= S3R_MAX_K || L + i >= p.cap || n < 0 || n > p.sel_stride) {
    if (c == 0 && tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int A = n + i + 1;
  const int nch = draft_nchunks(A);
  if (c >= nch) return;
  const int start = c * kDraftChunk;
  const int end = c == nch - 1 ? A : start + kDraftChunk;
  const int* ptab = p.page_table + (size_t)r * p.max_pages;
  const int64_t npages = p.num_pages;
  const size_t new_off = (size_t)r * p.kv_stride + (size_t)kvh * D;   // this token in k_new / v_new

  // This step's token enters the cache at position L+i (read below from k_new / v_new).
  if (c == 0 && tid < CPR) {
    const int pos = L + i;
    const int page = ptab[pos >> 4];
    if (page < 0 || page >= npages) {
      set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    } else {
      const size_t dst = (((size_t)page * Hkv + kvh) * kPage + (pos & 15)) * D + tid * 8;
      *reinterpret_cast<uint4*>(p.k_pool + dst) =
          *reinterpret_cast<const uint4*>(p.k_new + new_off + tid * 8);
      *reinterpret_cast<uint4*>(p.v_pool + dst) =
          *reinterpret_cast<const uint4*>(p.v_new + new_off + tid * 8);
    }
  }

  // The query rows first (their loads overlap the index work below).
  WarpAttn<D, NTW> wa;
  wa.init();
  wa.load_q(0, lane, [&](int rr) -> const __nv_bfloat16* {
    return rr < G ? p.q + (size_t)r * p.q_stride + (size_t)(kvh * G + rr) * D : nullptr;
  });

  // Element offsets of the chunk's rows: >= 0 pool offset, -1 zeros, -2 this step's token.
  // The positions from the indices loaded above, then all page ids in one round trip.
  int pos[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int a = start + tid + 128 * u;
    pos[u] = a < end ? (a < n ? selv[u] : L + (a - n)) : -1;
  }
  int page[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int a = start + tid + 128 * u;
    const bool look = a < end && pos[u] >= 0 && pos[u] < L + i;   // a committed position
    page[u] = look ? ptab[pos[u] >> 4] : -1;
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int a = start + tid + 128 * u;
    int64_t off = -1;
    if (a < end) {
      if (a < n && (pos[u] < 0 || pos[u] >= L)) {
        set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
      } else if (pos[u] == L + i) {
        off = -2;
      } else if (page[u] < 0 || page[u] >= npages) {
        set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
      } else {
        off = (((int64_t)page[u] * Hkv + kvh) * kPage + (pos[u] & 15)) * D;
      }
    }
    rowoff[tid + 128 * u] = off;
  }
  __syncthreads();

  const int ntiles = (end - start + kTile - 1) / kTile;
  const uint32_t sbase = smem_u32(smem);
  auto load_tile = [&](int it) {
    const uint32_t kdst = sbase + (it % kDraftStages) * STAGE, vdst = kdst + kTile * D * 2;
    for (int idx = tid; idx < kTile * CPR; idx += blockDim.x) {
      const int row = idx / CPR, ch = idx - row * CPR;
      const int64_t off = rowoff[it * kTile + row];
      const __nv_bfloat16 *ks, *vs;
      int bytes = 16;
      if (off >= 0) {
        ks = p.k_pool + off + ch * 8;
        vs = p.v_pool + off + ch * 8;
      } else if (off == -2) {
        ks = p.k_new + new_off + ch * 8;
        vs = p.v_new + new_off + ch * 8;
      } else {
        ks = p.k_new + new_off;   // any valid address; nothing is read
        vs = p.v_new + new_off;
        bytes = 0;
      }
      cp_async16(kdst + swz(row, ch), ks, bytes);
      cp_async16(vdst + swz(row, ch), vs, bytes);
    }
  };

#pragma unroll
  for (int s = 0; s < kDraftStages - 1; ++s) {
    if (s < ntiles) load_tile(s);
    cp_async_commit();
  }
  for (int it = 0; it < ntiles; ++it) {
    if (it + kDraftStages - 1 < ntiles) load_tile(it + kDraftStages - 1);
    cp_async_commit();
    cp_async_wait<kDraftStages - 1>();
    __syncthreads();
    const int t0 = start + it * kTile;
    const uint32_t kb = sbase + (it % kDraftStages) * STAGE, vb = kb + kTile * D * 2;
    const int row0 = warp * 16;
    if (t0 + row0 < end) {
      auto vis = [&](int tr, int, int) -> bool { return t0 + tr < end; };
      auto nocap = [](int, int, float, float) {};
      if (t0 + kTile <= end)
        wa.template step<false>(kb, vb, row0, lane, p.scale, vis, nocap);
      else
        wa.template step<true>(kb, vb, row0, lane, p.scale, vis, nocap);
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  wa.finish_sums();
  float* redO = reinterpret_cast<float*>(smem);
  float* redM = redO + 4 * RW * (D + 4);
  float* redL = redM + 4 * RW;
  wa.store_shared(redO, redM, redL, warp, lane);
  __syncthreads();
  auto out_row = [&](int row) { return p.out + ((size_t)r * p.Hq + kvh * G + row) * D; };
  auto lse_row = [&](int row) -> float* { return p.lse ? p.lse + (size_t)r * p.Hq + kvh * G + row : nullptr; };
  __shared__ float fw[4 * RW], Mrow[RW], Lrow[RW];
  slice_weights<RW>(redM, redL, G, fw, Mrow, Lrow, tid);
  if (nch == 1) {
    slices_to_output<D, RW>(redO, fw, Mrow, Lrow, G, out_row, lse_row, tid, blockDim.x);
    return;
  }
  const size_t rec_floats = (size_t)RW * (D + 2);
  float* recs = p.part + ((size_t)r * Hkv + kvh) * p.nchunk_max * rec_floats;
  slices_to_record<D, RW>(redO, fw, Mrow, Lrow, G, recs + c * rec_floats, tid, blockDim.x);

  if (!last_of(p.tickets + (size_t)r * Hkv + kvh, nch, s_flag)) return;
  if (nch <= kDraftFastMerge) {
    combine_few_records<D, RW>(recs, rec_floats, nch, G, out_row, lse_row, tid, blockDim.x);
    return;
  }
  __shared__ float wts[32 * RW];
  combine_records<D>(recs, rec_floats, nch, G, RW, wts, 32 * RW, out_row, lse_row, tid, blockDim.x);
}

template <int D>
static int launch_draft_d(const DraftParams& p, int batch, cudaStream_t stream) {
  const size_t smem = 1024 + kDraftStages * 2 * kTile * D * 2 + kDraftSpan * 8 + 64;
  static std::atomic<uint64_t> attr_done{0};
  if (cuda_status(ensure_smem_attr(draft_kernel<D>, (int)smem, attr_done), "cudaFuncSetAttribute") != S3R_OK)
    return S3R_ERR_CUDA;
  dim3 grid(p.Hkv, batch, p.nchunk_max);
  launch_pdl(draft_kernel<D>, grid, 128, smem, stream, p);
  return cuda_status(cudaGetLastError(), __func__);
}

int launch_draft(const DraftParams& p, int D, int batch, int /*num_sms*/, cudaStream_t stream, int* launches) {
  *launches = 0;
  int st = S3R_ERR_UNSUPPORTED;
  if (D == 128) st = launch_draft_d<128>(p, batch, stream);
  if (D == 64) st = launch_draft_d<64>(p, batch, stream);
  if (st == S3R_OK) *launches = 1;
  return st;
}

int draft_chunks(int sel_stride) { return (sel_stride + S3R_MAX_K + 1 + kDraftChunk - 1) / kDraftChunk; }

size_t draft_partial_bytes(int num_requests, int Hkv, int sel_stride, int D) {
  return align_up((size_t)num_requests * Hkv * draft_chunks(sel_stride) * 8 * (D + 2) * 4, 256);
}

}  // namespace s3r
