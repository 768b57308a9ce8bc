// Sparse KV selection as a block-wide radix select.
//
// What it computes ([Explainer] Jargon, sparse attention budget: the newest positions plus
// those the verifier attended to most; walkthrough: refreshed after every round): for
// request r at committed length L and KV head h, n = clamp(ceil(L * bp / 1e4), W', L)
// positions, W' = min(W, L): the W' newest plus the n - W' highest-scored positions
// j < L - W', ties to the lower j, ascending.
//
// Page-granular variant ([Explainer] walkthrough: "top-scoring pages"): the units are the
// 16-position pages wholly before the window, each scored by the fp32 sum of its positions'
// scores added in position order; the pages holding the W' newest positions are kept whole;
// ceil(n / 16) pages in all (at least the window's); every position of a chosen page below L
// is emitted, ascending, so the count is at most n + 15.
//
// One CTA of 1024 threads per (KV head, request), the CTAs taking the pairs ranked by
// request length so that the two on an SM hold a long and a short set. Scores sigma_j = sum over the G*(k+1)
// verify rows of exp(logit - lse) are computed once into shared memory as order-preserving
// uint32 keys; MSB-first histogram passes over digits of 11, 11 and 10 bits (shared atomics,
// one block scan over the bins per pass; the first pass is counted while the keys are
// loaded) find the M-th largest score's digits and how many ties to keep, stopping early
// once the bin that holds it is taken whole; a final pass compacts the chosen indices in
// increasing order, each thread over its own contiguous run of positions.
#include "common.cuh"
#include "kernels.h"

namespace s3r {

constexpr int kSelectThreads = 1024;
constexpr int kSelectMaxN = 49152;   // non-window positions held in shared memory
constexpr int kSelectBins = 2048;    // digits of up to 11 bits
constexpr int kSelectRankMax = 1024; // requests per launch ranked for the CTA pairing

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;              // -0 and +0 compare equal
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum of `v` in thread order (1024 threads); `wsum` holds 32
// ints of scratch. Ends with a barrier.
__device__ __forceinline__ int block_excl_scan(int v, int* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int t = wsum[lane];
    int ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(kFull, ti, o);
      if (lane >= o) ti += n;
    }
    wsum[lane] = ti - t;
  }
  __syncthreads();
  const int r = wsum[warp] + incl - v;
  __syncthreads();
  return r;
}

template <int P>
__global__ void __launch_bounds__(kSelectThreads, 2) select_kernel(const SelectParams p) {
  pdl_wait();
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[kSelectBins];
  __shared__ int wsum[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining, s_whole;

  const int tid = threadIdx.x;
  int kvh = blockIdx.x, bl = blockIdx.y;
  // Balance: the block scheduler places CTA c (linear index) and CTA c + num_sms on the
  // same SM, and a CTA's work grows with its request's length. With the requests ranked
  // by length (longest first, ties to the lower slot) and pairs numbered rank * Hkv + head,
  // CTA c < num_sms takes pair c and CTA num_sms + j takes pair total - 1 - j, so one SM's
  // two CTAs hold a long and a short set. Up to kSelectRankMax requests per launch.
  const int nb = gridDim.y, total = nb * p.Hkv;
  if (total > p.num_sms && p.num_sms > 0 && nb <= kSelectRankMax) {
    __shared__ int s_len[kSelectRankMax];
    __shared__ int s_slot;
    for (int j = tid; j < nb; j += blockDim.x) {
      const int rj = p.req_ids ? p.req_ids[j] : j;
      s_len[j] = (rj >= 0 && rj < p.num_requests) ? p.seq_lens[rj] : -1;
    }
    __syncthreads();
    const int c = blockIdx.x + p.Hkv * blockIdx.y;
    const int t = c < p.num_sms ? c : total - 1 - (c - p.num_sms);
    const int want = t / p.Hkv;
    for (int j = tid; j < nb; j += blockDim.x) {
      const int Lj = s_len[j];
      int rank = 0;
      for (int q = 0; q < nb; ++q) rank += (s_len[q] > Lj) || (s_len[q] == Lj && q < j);
      if (rank == want) s_slot = j;
    }
    __syncthreads();
    bl = s_slot;
    kvh = t - want * p.Hkv;
  }
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) {
    if (kvh == 0 && tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int L = p.seq_lens[r];
  if (L < 0 || L > p.score_stride) {
    if (tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  int n = (int)(((int64_t)L * p.budget_bp + 9999) / 10000);
  const int w = min(p.window, L);
  n = min(max(n, w), L);
  // units: positions (P = 1) or pages (P = 16); M of the N candidate units are chosen, the
  // window's units start at position wstart, cnt positions are emitted
  int M, N, wstart;
  if constexpr (P == 1) {
    M = n - w;
    N = L - w;
    wstart = N;
  } else {
    N = (L - w) / P;
    const int win_pages = (L + P - 1) / P - N;
    M = max((n + P - 1) / P - win_pages, 0);
    wstart = N * P;
  }
  const int cnt = M * P + (L - wstart);
  if (cnt > p.sel_stride) {
    if (tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  if (M > 0 && N > kSelectMaxN) {
    if (tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  int32_t* out = p.sel_idx + ((size_t)r * p.Hkv + kvh) * p.sel_stride;
  for (int j = tid; j < L - wstart; j += blockDim.x) out[M * P + j] = wstart + j;
  if (tid == 0) p.sel_count[(size_t)r * p.Hkv + kvh] = cnt;
  if (M == 0) return;
  for (int b = tid; b < kSelectBins; b += blockDim.x) hist[b] = 0;
  __syncthreads();

  // ---- scores -> order-preserving keys in shared memory, with the histogram of their top
  // 11 bits (the first digit)
  constexpr int kShift0 = 32 - 11;
  bool bad = false;
  const float* srow = p.scores + ((size_t)r * p.Hkv + kvh) * p.score_stride;
  int jv = 0;   // positions below jv were loaded as 16-byte vectors
  if constexpr (P == 1) {
    if ((reinterpret_cast<uintptr_t>(srow) & 15u) == 0) {
      // every thread has kU 16-byte loads in flight before it converts them
      constexpr int kU = 4;
      const int n4 = N >> 2;
      const float4* s4 = reinterpret_cast<const float4*>(srow);
      for (int b0 = 0; b0 < n4; b0 += kU * kSelectThreads) {
        float4 v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int i4 = b0 + u * kSelectThreads + tid;
          v[u] = i4 < n4 ? __ldg(s4 + i4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int i4 = b0 + u * kSelectThreads + tid;
          if (i4 < n4) {
            float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t kk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (!isfinite(x[e])) {
                bad = true;
                x[e] = -INFINITY;
              }
              kk[e] = order_key(x[e]);
              atomicAdd(&hist[kk[e] >> kShift0], 1u);
            }
            *reinterpret_cast<uint4*>(keys + 4 * i4) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
          }
        }
      }
      jv = n4 * 4;
    }
  }
  for (int j = jv + tid; j < N; j += blockDim.x) {
    float sigma;
    if constexpr (P == 1) {
      sigma = srow[j];
      if (!isfinite(sigma)) {
        bad = true;
        sigma = -INFINITY;
      }
    } else {
      const float* sp = srow + (size_t)j * P;
      sigma = sp[0];
      bool fin = isfinite(sigma);
      for (int t = 1; t < P; ++t) {
        const float x = sp[t];
        fin = fin && isfinite(x);
        sigma = __fadd_rn(sigma, x);   // position order, one rounding per add
      }
      if (!fin) {
        bad = true;
        sigma = -INFINITY;
      }
    }
    const uint32_t key = order_key(sigma);
    keys[j] = key;
    atomicAdd(&hist[key >> kShift0], 1u);
  }
  if (bad) set_error(p.err, S3R_ERR_NONFINITE);
  __syncthreads();

  // ---- radix select of the M-th largest key, MSB-first in digits of 11, 11 and 10 bits.
  // A pass histograms the digit of the keys that match the prefix chosen so far (the first
  // pass was counted above); one block scan over the bins from the top finds the bin holding
  // the remaining-th largest. When that bin holds exactly the keys still wanted, all of it is
  // taken and the lower digits need no pass.
  uint32_t prefix = 0u, mask = 0u;
  int remaining = M;
  int shift = kShift0, width = 32 - kShift0;
#pragma unroll 1
  while (true) {
    const int nb = 1 << width;
    // thread t owns bins 2047-2t and 2046-2t of the 2048-bin view (descending); bins at or
    // above nb are empty
    int h[2], local = 0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int bin = kSelectBins - 1 - 2 * tid - q;
      h[q] = bin < nb ? (int)hist[bin] : 0;
      local += h[q];
    }
    const int before = block_excl_scan(local, wsum);
    if (before < remaining && remaining <= before + local) {
      int cum = before;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (cum + h[q] >= remaining) {
          s_prefix = prefix | ((uint32_t)(kSelectBins - 1 - 2 * tid - q) << shift);
          s_remaining = remaining - cum;
          s_whole = (remaining - cum == h[q]);
          break;
        }
        cum += h[q];
      }
    }
    __syncthreads();
    prefix = s_prefix;
    remaining = s_remaining;
    mask |= (uint32_t)(nb - 1) << shift;
    if (shift == 0 || s_whole) break;
    width = shift < 11 ? shift : 11;
    shift -= width;
    for (int b = tid; b < kSelectBins; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const uint32_t dmask = (uint32_t)((1 << width) - 1);
    const int n4 = N >> 2;
    const uint4* k4 = reinterpret_cast<const uint4*>(keys);
    for (int i4 = tid; i4 < n4; i4 += blockDim.x) {
      const uint4 kv = k4[i4];
      if ((kv.x & mask) == prefix) atomicAdd(&hist[(kv.x >> shift) & dmask], 1u);
      if ((kv.y & mask) == prefix) atomicAdd(&hist[(kv.y >> shift) & dmask], 1u);
      if ((kv.z & mask) == prefix) atomicAdd(&hist[(kv.z >> shift) & dmask], 1u);
      if ((kv.w & mask) == prefix) atomicAdd(&hist[(kv.w >> shift) & dmask], 1u);
    }
    for (int j = 4 * n4 + tid; j < N; j += blockDim.x) {
      const uint32_t key = keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
  }
  // Keys whose resolved digits exceed the prefix are taken, and the first `remaining` keys
  // (in position order) whose resolved digits equal it; unresolved low digits (a bin taken
  // whole) do not matter.
  const uint32_t thr = prefix;
  const int need_eq = remaining;

  // ---- ordered compaction: thread t owns the run of positions [t per, t per + per), read
  // as 16-byte vectors (per / 4 odd, so the eight threads of a quarter-warp hit distinct
  // banks); two block scans give each thread the equal keys before its run and its first
  // output slot, then every thread writes its picks in position order
  int per = ((N + kSelectThreads - 1) / kSelectThreads + 3) & ~3;
  if ((per & 7) == 0) per += 4;
  const int j0 = min(tid * per, N), j1 = min(N, j0 + per);
  int gt_t = 0, eq_t = 0;
  for (int jb = j0; jb < j1; jb += 4) {
    const uint4 kv = *reinterpret_cast<const uint4*>(keys + jb);
    const uint32_t kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t key = kk[e] & mask;
      const bool in = jb + e < j1;
      gt_t += in && key > thr;
      eq_t += in && key == thr;
    }
  }
  const int eq_before = block_excl_scan(eq_t, wsum);
  int base = block_excl_scan(gt_t + min(max(need_eq - eq_before, 0), eq_t), wsum);
  int eqb = eq_before;
  for (int jb = j0; jb < j1; jb += 4) {
    const uint4 kv = *reinterpret_cast<const uint4*>(keys + jb);
    const uint32_t kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t key = kk[e] & mask;
      if (jb + e < j1 && (key > thr || (key == thr && eqb < need_eq))) {
        int32_t* o = out + (size_t)base * P;
        for (int t = 0; t < P; ++t) o[t] = (jb + e) * P + t;
        ++base;
      }
      eqb += (jb + e < j1 && key == thr);
    }
  }
}

// ---- scores from a verify's logits: sigma_j = sum over the G*(k+1) rows of
// 2^(logit * log2(e) - lse * log2(e)) for every non-window position j < L - min(W, L),
// written as fp32 [NR][Hkv][cap]. A flat grid over (block of 1024 positions, KV head,
// request) at full occupancy: the logits of one row are contiguous over positions, each
// thread takes 4 positions and keeps 8 rows' 16-byte loads in flight.
constexpr int kSigmaThreads = 256;
constexpr int kSigmaPos = 4 * kSigmaThreads;

__global__ void __launch_bounds__(kSigmaThreads) sigma_kernel(const SelectParams p) {
  pdl_wait();
  __shared__ float lse2[S3R_MAX_ROWS];
  const int kvh = blockIdx.y, bl = blockIdx.z;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) {
    // reported by the select kernel on its path; here for the scores-only call
    if (p.window == 0 && blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int L = p.seq_lens[r];
  if (L < 0 || L > p.cap || L > p.sigma_stride) {
    // reported by the select kernel on its path; here for the scores-only call
    if (p.window == 0 && blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int N = L - min(p.window, L);
  const int j0 = blockIdx.x * kSigmaPos;
  if (j0 >= N) return;
  for (int row = threadIdx.x; row < p.R; row += blockDim.x) {
    const int t = row / p.G, g = row - t * p.G;
    lse2[row] = p.lse[((size_t)r * p.T + t) * p.Hq + kvh * p.G + g] * kLog2e;
  }
  __syncthreads();
  const int j4 = j0 + 4 * (int)threadIdx.x;
  if (j4 >= N) return;
  const float* base = p.logits + ((size_t)r * p.Hkv + kvh) * (size_t)p.R * p.cap + j4;
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  for (int row0 = 0; row0 < p.R; row0 += 8) {
    float4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (row0 + u < p.R) x[u] = __ldg(reinterpret_cast<const float4*>(base + (size_t)(row0 + u) * p.cap));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (row0 + u >= p.R) break;
      const float l2 = lse2[row0 + u];
      acc0 += ex2(fmaf(x[u].x, kLog2e, -l2));
      acc1 += ex2(fmaf(x[u].y, kLog2e, -l2));
      acc2 += ex2(fmaf(x[u].z, kLog2e, -l2));
      acc3 += ex2(fmaf(x[u].w, kLog2e, -l2));
    }
  }
  float* out = p.sigma_buf + ((size_t)r * p.Hkv + kvh) * p.sigma_stride + j4;
  if (j4 + 4 <= N) {
    *reinterpret_cast<float4*>(out) = make_float4(acc0, acc1, acc2, acc3);
  } else {
    const float sg[4] = {acc0, acc1, acc2, acc3};
    for (int q = 0; q < N - j4; ++q) out[q] = sg[q];
  }
}

int launch_sigma(const SelectParams& p, int batch, cudaStream_t stream) {
  dim3 g((p.cap + kSigmaPos - 1) / kSigmaPos, p.Hkv, batch);
  launch_pdl(sigma_kernel, g, kSigmaThreads, 0, stream, p);
  return cuda_status(cudaGetLastError(), "sigma_kernel");
}

size_t select_sigma_bytes(int num_requests, int Hkv, int cap) {
  return align_up((size_t)num_requests * Hkv * cap * 4, 256);
}

int launch_select(const SelectParams& p, int batch, cudaStream_t stream, int* launches) {
  *launches = 0;
  SelectParams q = p;
  if (p.logits) {
    q.sigma_stride = p.cap;
    dim3 g((p.cap + kSigmaPos - 1) / kSigmaPos, p.Hkv, batch);
    launch_pdl(sigma_kernel, g, kSigmaThreads, 0, stream, q);
    if (cuda_status(cudaGetLastError(), "sigma_kernel") != S3R_OK) return S3R_ERR_CUDA;
    ++*launches;
    q.logits = nullptr;
    q.scores = p.sigma_buf;
    q.score_stride = p.cap;
  }
  const int lim = q.score_stride;
  const int nmax = lim < kSelectMaxN ? lim : kSelectMaxN;
  // whole 16-byte vectors: the last one may reach 3 keys past the set
  const size_t smem = align_up((size_t)(nmax > 0 ? nmax : 1), 4) * 4;
  static std::atomic<uint64_t> attr_tok{0}, attr_page{0};
  if (cuda_status(ensure_smem_attr(select_kernel<1>, kSelectMaxN * 4, attr_tok), "cudaFuncSetAttribute") != S3R_OK ||
      cuda_status(ensure_smem_attr(select_kernel<S3R_PAGE_SIZE>, kSelectMaxN * 4, attr_page),
                  "cudaFuncSetAttribute") != S3R_OK)
    return S3R_ERR_CUDA;
  dim3 grid(q.Hkv, batch);
  if (p.page == S3R_PAGE_SIZE)
    launch_pdl(select_kernel<S3R_PAGE_SIZE>, grid, kSelectThreads, smem, stream, q);
  else
    launch_pdl(select_kernel<1>, grid, kSelectThreads, smem, stream, q);
  const int st = cuda_status(cudaGetLastError(), __func__);
  if (st == S3R_OK) ++*launches;
  return st;
}

}  // namespace s3r
