// Sparse KV selection as a block-wide radix select.
//
// What it computes ([Explainer] Jargon, sparse attention budget: the newest positions plus
// those the verifier attended to most; walkthrough: refreshed after every round): for
// request r at committed length L and KV head h, n = clamp(ceil(L * bp / 1e4), W', L)
// positions, W' = min(W, L): the W' newest plus the n - W' highest-scored positions
// j < L - W', ties to the lower j, ascending.
//
// One CTA of 1024 threads per (KV head, request). Scores sigma_j = sum over the G*(k+1)
// verify rows of exp(logit - lse) are computed once into shared memory as order-preserving
// uint32 keys; four 8-bit MSB-first histogram passes (warp-aggregated shared atomics) find
// the exact key of the M-th largest score and how many ties at that key to keep; a final
// pass compacts the chosen indices in increasing order with ballot-based block scans.
#include "common.cuh"
#include "kernels.h"

namespace s3r {

constexpr int kSelectThreads = 1024;
constexpr int kSelectMaxN = 49152;   // non-window positions held in shared memory

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f == 0.f) f = 0.f;              // -0 and +0 compare equal
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide prefix count of `flag`; also returns the block total.
__device__ __forceinline__ int block_excl_count(bool flag, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned b = __ballot_sync(kFull, flag);
  const int in_warp = __popc(b & ((1u << lane) - 1u));
  if (lane == 0) warp_tot[warp] = __popc(b);
  __syncthreads();
  int before = 0, tot = 0;
  const int nw = blockDim.x >> 5;
  for (int w = 0; w < nw; ++w) {
    const int v = warp_tot[w];
    before += (w < warp) ? v : 0;
    tot += v;
  }
  __syncthreads();
  total = tot;
  return before + in_warp;
}

__global__ void __launch_bounds__(kSelectThreads) select_kernel(const SelectParams p) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ float lse_s[S3R_MAX_ROWS];
  __shared__ int warp_tot[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;

  const int tid = threadIdx.x, lane = tid & 31;
  const int kvh = blockIdx.x, bl = blockIdx.y;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  const int L = p.seq_lens[r];
  const int lim = p.logits ? p.cap : p.score_stride;
  if (L < 0 || L > lim) {
    if (tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  int n = (int)(((int64_t)L * p.budget_bp + 9999) / 10000);
  const int w = min(p.window, L);
  n = min(max(n, w), L);
  if (n > p.sel_stride) {
    if (tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int M = n - w, N = L - w;
  if (M > 0 && N > kSelectMaxN) {
    if (tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  int32_t* out = p.sel_idx + ((size_t)r * p.Hkv + kvh) * p.sel_stride;
  for (int j = tid; j < w; j += blockDim.x) out[M + j] = N + j;
  if (tid == 0) p.sel_count[(size_t)r * p.Hkv + kvh] = n;
  if (M == 0) return;

  // ---- scores -> keys
  if (p.logits) {
    for (int row = tid; row < p.R; row += blockDim.x) {
      const int t = row / p.G, g = row - t * p.G;
      lse_s[row] = p.lse[((size_t)r * p.T + t) * p.Hq + kvh * p.G + g];
    }
    __syncthreads();
  }
  bool bad = false;
  for (int j = tid; j < N; j += blockDim.x) {
    float sigma;
    if (p.logits) {
      // the G*(k+1) logits of position j are contiguous: [..][cap][R]
      const float* lg = p.logits + (((size_t)r * p.Hkv + kvh) * p.cap + j) * p.R;
      float acc = 0.f;
      if ((p.R & 3) == 0) {
        for (int row = 0; row < p.R; row += 4) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(lg + row));
          acc += expf(x.x - lse_s[row]) + expf(x.y - lse_s[row + 1]) +
                 expf(x.z - lse_s[row + 2]) + expf(x.w - lse_s[row + 3]);
        }
      } else if ((p.R & 1) == 0) {
        for (int row = 0; row < p.R; row += 2) {
          const float2 x = __ldg(reinterpret_cast<const float2*>(lg + row));
          acc += expf(x.x - lse_s[row]) + expf(x.y - lse_s[row + 1]);
        }
      } else {
        for (int row = 0; row < p.R; ++row) acc += expf(__ldg(lg + row) - lse_s[row]);
      }
      sigma = acc;
    } else {
      sigma = p.scores[((size_t)r * p.Hkv + kvh) * p.score_stride + j];
    }
    if (!isfinite(sigma)) {
      bad = true;
      sigma = -INFINITY;
    }
    keys[j] = order_key(sigma);
  }
  if (bad) set_error(p.err, S3R_ERR_NONFINITE);
  __syncthreads();

  // ---- radix select of the M-th largest key
  uint32_t prefix = 0, mask = 0;
  int remaining = M;
  const int Nround = (N + blockDim.x - 1) / blockDim.x * blockDim.x;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    for (int j = tid; j < Nround; j += blockDim.x) {
      const uint32_t key = j < N ? keys[j] : 0u;
      const bool part = j < N && (key & mask) == prefix;
      const uint32_t digit = (key >> shift) & 255u;
      const unsigned peers = __match_any_sync(kFull, part ? digit : (0x100u + lane));
      if (part && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins 255-8l .. 248-8l (descending)
      uint32_t loc = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) loc += hist[255 - 8 * lane - q];
      uint32_t incl = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - loc;
      const unsigned hit = __ballot_sync(kFull, incl >= (uint32_t)remaining);
      const int owner = __ffs(hit) - 1;
      if (lane == owner) {
        uint32_t cum = excl;
        int dsel = 248 - 8 * lane;
        for (int q = 0; q < 8; ++q) {
          const int bin = 255 - 8 * lane - q;
          if (cum + hist[bin] >= (uint32_t)remaining) {
            dsel = bin;
            break;
          }
          cum += hist[bin];
        }
        s_prefix = prefix | ((uint32_t)dsel << shift);
        s_remaining = remaining - (int)cum;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    remaining = s_remaining;
    mask |= 255u << shift;
  }
  // prefix is the key of the M-th largest score; `remaining` keys equal to it are kept.
  const uint32_t thr = prefix;
  const int need_eq = remaining;

  // ---- ordered compaction
  int base = 0, eq_seen = 0;
  for (int j0 = 0; j0 < N && base < M; j0 += blockDim.x) {
    const int j = j0 + tid;
    const uint32_t key = j < N ? keys[j] : 0u;
    const bool gt = j < N && key > thr;
    const bool eq = j < N && key == thr;
    int eq_tot, take_tot;
    const int eq_rank = eq_seen + block_excl_count(eq, warp_tot, eq_tot);
    const bool take = gt || (eq && eq_rank < need_eq);
    const int at = base + block_excl_count(take, warp_tot, take_tot);
    if (take) out[at] = j;
    base += take_tot;
    eq_seen += eq_tot;
  }
}

int launch_select(const SelectParams& p, int batch, cudaStream_t stream) {
  const int lim = p.logits ? p.cap : p.score_stride;
  const int nmax = lim < kSelectMaxN ? lim : kSelectMaxN;
  const size_t smem = (size_t)(nmax > 0 ? nmax : 1) * 4;
  static bool attr_done = false;
  if (!attr_done) {
    if (cuda_status(cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSelectMaxN * 4), "cudaFuncSetAttribute") != S3R_OK)

      return S3R_ERR_CUDA;
    attr_done = true;
  }
  dim3 grid(p.Hkv, batch);
  select_kernel<<<grid, kSelectThreads, smem, stream>>>(p);
  return cuda_status(cudaGetLastError(), __func__);
}

}  // namespace s3r
