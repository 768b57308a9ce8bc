// Draft-token sampling, exact speculative sampling, round commit and Philox uniforms.
//
// What they compute ([News] Interpretation and [Explainer] Jargon, exact speculative
// sampling: accept a draft or draw from the residual distribution so that emitted tokens
// follow the dense policy): softmax normalisers of the draft / target rows, the accept
// tests u * q(d) < p(d), and inverse-CDF draws from q, from max(0, p - q) or from p.
//
// The vocabulary is split into chunks of 8192 entries. A pass over (chunk, row, request)
// produces (max, sum exp(x - max)) per chunk with fp32 exponentials and fp64 sums; the last
// CTA of a request merges the chunks (ticket, no spinning) and decides. A draw first finds
// the chunk holding u * Z from the chunk sums, then the warp holding it (warp totals in
// order), then, inside that warp's 1024 entries, the row of 32 and the entry.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace s3r {

constexpr int kSampThreads = 256;

struct MS {
  float m;
  float pad;
  double s;
};
static_assert(sizeof(MS) == kSamplePartialBytes, "partial record size");

struct SpecPlan {
  int type;      // 0: residual of row j, 1: target row j
  int row;
  int a;         // accepted drafts
  int pad;
  float mp, mq;
  double zp, zq, u;
};

// (max, sum 2^((x - max) log2 e)) of this thread's share of row[v0 .. v1): up to 32 entries,
// as eight 16-byte loads (v0 + 4 (t + 256 j)) when the range is 16-byte aligned, else as
// strided scalars. NaN and +inf are flagged and count as probability 0; -inf is a valid
// zero-probability logit.
__device__ __forceinline__ void thread_ms(const float* row, int v0, int v1, float& m, float& s,
                                          bool& bad) {
  float x[32];
  const bool vec = ((reinterpret_cast<uintptr_t>(row + v0) & 15u) == 0) && (((v1 - v0) & 3) == 0);
  if (vec) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int v = v0 + 4 * ((int)threadIdx.x + kSampThreads * j);
      float4 q = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (v < v1) q = __ldg(reinterpret_cast<const float4*>(row + v));
      x[4 * j] = q.x;
      x[4 * j + 1] = q.y;
      x[4 * j + 2] = q.z;
      x[4 * j + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int v = v0 + (int)threadIdx.x + kSampThreads * j;
      x[j] = v < v1 ? __ldg(row + v) : -INFINITY;
    }
  }
  m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (isnan(x[j]) || x[j] == INFINITY) {
      bad = true;
      x[j] = -INFINITY;
    }
    m = fmaxf(m, x[j]);
  }
  s = 0.f;
  if (m != -INFINITY) {
    const float mb = m * kLog2e;
#pragma unroll
    for (int j = 0; j < 32; ++j) s += ex2(fmaf(x[j], kLog2e, -mb));
  }
}

// Block reduction of per-thread (max, sum) pairs; the result is valid in thread 0.
__device__ MS block_ms(float m, float s) {
  __shared__ float sm[kSampThreads / 32];
  __shared__ float ss[kSampThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float mw = warp_max(m);
  float sw = (m == -INFINITY) ? 0.f : s * ex2((m - mw) * kLog2e);
#pragma unroll
  for (int o = 16; o; o >>= 1) sw += __shfl_xor_sync(kFull, sw, o);
  if (lane == 0) {
    sm[warp] = mw;
    ss[warp] = sw;
  }
  __syncthreads();
  MS r{-INFINITY, 0.f, 0.0};
  if (threadIdx.x == 0) {
    for (int w = 0; w < kSampThreads / 32; ++w) r.m = fmaxf(r.m, sm[w]);
    for (int w = 0; w < kSampThreads / 32; ++w)
      if (sm[w] != -INFINITY) r.s += (double)ss[w] * (double)ex2((sm[w] - r.m) * kLog2e);
  }
  return r;
}

// Merge one row's chunk partials with one warp: lane q loads partial q (and q + 32), so
// the loads are one round trip, not one per chunk. Writes the chunk weights
// csum[q] = s_q 2^((m_q - M) log2 e) (fp64) and returns the row maximum M on every lane.
__device__ __forceinline__ float merge_partials_warp(const MS* part, int nvch, double* csum) {
  const int lane = threadIdx.x & 31;
  float mq[2] = {-INFINITY, -INFINITY};
  double sq[2] = {0.0, 0.0};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int q = lane + 32 * h;
    if (q < nvch) {
      mq[h] = __ldcg(&part[q].m);
      sq[h] = __ldcg(&part[q].s);
    }
  }
  const float M = warp_max(fmaxf(mq[0], mq[1]));
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int q = lane + 32 * h;
    if (q < nvch) csum[q] = (mq[h] == -INFINITY) ? 0.0 : sq[h] * (double)exp2f((mq[h] - M) * kLog2e);
  }
  return M;
}

__device__ double block_sum_d(double v) {
  __shared__ double sd[kSampThreads / 32];
  __shared__ double tot;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum_d(v);
  if (lane == 0) sd[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kSampThreads / 32; ++w) t += sd[w];
    tot = t;
  }
  __syncthreads();
  const double r = tot;
  __syncthreads();
  return r;
}

// Inverse-CDF search inside [v0, v1) (at most kVocabChunk entries): smallest v with
// target < base + C_v, C the inclusive running sum of weight(v). Warp w takes the 1024
// entries v0 + 1024 w + 32 m + lane (m = 0..31: coalesced loads, weights kept in
// registers); the warps' totals, in order, find the warp holding the target; that warp
// reduces its 32 rows of 32 entries with a butterfly (lane m ends with row m's sum),
// scans the rows, then the lanes of the chosen row. Returns -1 if the target lies past the
// chunk; `base` then moves to the chunk's end.
// `mrg` receives the distance of the target to the nearer edge of the drawn token's cell
// [C_{v-1}, C_v) (0 where rounding carried the target past the last entry).
template <class W>
__device__ int chunk_search(int v0, int v1, double target, double& base, double& mrg, W weight) {
  __shared__ double wtot_s[kSampThreads / 32];
  __shared__ int s_tok;
  __shared__ double s_mrg;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int wb = v0 + warp * 1024;
  float w[32];
  float part = 0.f;
#pragma unroll
  for (int m = 0; m < 32; ++m) {
    const int v = wb + 32 * m + lane;
    w[m] = v < v1 ? weight(v) : 0.f;
    part += w[m];
  }
  const double wt = warp_sum_d((double)part);
  if (lane == 0) wtot_s[warp] = wt;
  if (threadIdx.x == 0) {
    s_tok = -1;
    s_mrg = 0.0;
  }
  __syncthreads();
  double lo = base, total = 0.0;
  for (int q = 0; q < kSampThreads / 32; ++q) {
    if (q < warp) lo += wtot_s[q];
    total += wtot_s[q];
  }
  if (wt > 0.0 && target >= lo && target < lo + wt) {
    // butterfly (in place): afterwards lane l holds row l's total in w[0]
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
      const bool up = (lane & k) != 0;
#pragma unroll
      for (int i = 0; i < k; ++i) {
        const float send = up ? w[i] : w[i + k];
        const float keep = up ? w[i + k] : w[i];
        w[i] = keep + __shfl_xor_sync(kFull, send, k);
      }
    }
    const double rs = w[0];
    double incl = rs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double t = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += t;
    }
    // row: the first with target < lo + (rows up to and including it)
    const unsigned rowhit = __ballot_sync(kFull, rs > 0.0 && target < lo + incl);
    int tok = -1;
    double m = 0.0;
    if (rowhit) {
      const int mr = __ffs(rowhit) - 1;
      const double rbase = lo + __shfl_sync(kFull, incl - rs, mr);
      const int vx = wb + 32 * mr + lane;   // the row's weights again (same values)
      const float x = vx < v1 ? weight(vx) : 0.f;
      double li = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(kFull, li, o);
        if (lane >= o) li += t;
      }
      const unsigned hit = __ballot_sync(kFull, x > 0.f && target < rbase + li);
      // rounding past the row's last entry: its last non-zero entry
      const unsigned nz = __ballot_sync(kFull, x > 0.f);
      const int ln = hit ? __ffs(hit) - 1 : 31 - __clz((int)nz);
      tok = wb + 32 * mr + ln;
      const double hi_e = rbase + li, lo_e = hi_e - (double)x;   // the lane's cell
      const double mine = fmin(target - lo_e, hi_e - target);
      m = hit ? __shfl_sync(kFull, mine, ln) : 0.0;
    } else {
      // rounding past the warp's last row: the last non-zero entry of the warp
      const unsigned nzr = __ballot_sync(kFull, rs > 0.0);
      const int mr = 31 - __clz((int)nzr);
      const int vx = wb + 32 * mr + lane;
      const float x = vx < v1 ? weight(vx) : 0.f;
      const unsigned nz = __ballot_sync(kFull, x > 0.f);
      tok = wb + 32 * mr + (31 - __clz((int)nz));
    }
    if (lane == 0) {
      s_tok = tok;
      s_mrg = m;
    }
  }
  __syncthreads();
  const int tok = s_tok;
  if (tok >= 0) mrg = s_mrg;
  base += total;
  __syncthreads();
  return tok;
}

// Last entry with non-zero weight in [0, V) (rounding fallback of a draw).
template <class W>
__device__ int last_nonzero(int V, W weight) {
  __shared__ int s_last;
  if (threadIdx.x == 0) s_last = -1;
  __syncthreads();
  for (int v = threadIdx.x; v < V; v += blockDim.x)
    if (weight(v) > 0.f) atomicMax(&s_last, v);
  __syncthreads();
  const int r = s_last;
  __syncthreads();
  return r < 0 ? V - 1 : r;
}

// Draw with target u * Z over weights whose chunk sums are csum[0..nvch).
// Inverse-CDF draw of target = u * Z from the chunk sums csum: thread 0 finds the chunk,
// stage(c0, n) brings that chunk's inputs into shared memory (ending with a barrier), and
// the search reads them there through sweight(v, c0); if rounding carries the target past
// the last chunk, the last token of nonzero weight (gweight reads global memory) is taken.
template <class Stage, class SW, class GW>
__device__ int draw_staged(int V, int nvch, const double* csum, double target, double& mrg,
                           Stage stage, SW sweight, GW gweight) {
  __shared__ int s_c;
  __shared__ double s_base;
  if (threadIdx.x == 0) {
    double cum = 0.0;
    int c = nvch;
    for (int i = 0; i < nvch; ++i) {
      if (target < cum + csum[i]) {
        c = i;
        break;
      }
      cum += csum[i];
    }
    s_c = c;
    s_base = cum;
  }
  __syncthreads();
  double base = s_base;
  int tok = -1;
  mrg = 0.0;
  for (int c = s_c; c < nvch && tok < 0; ++c) {
    const int c0 = c * kVocabChunk, cn = min(V - c0, kVocabChunk);
    __syncthreads();   // every thread is done with the shared buffers
    stage(c0, cn);
    tok = chunk_search(c0, c0 + cn, target, base, mrg, [&](int v) -> float { return sweight(v, c0); });
  }
  return tok >= 0 ? tok : last_nonzero(V, gweight);
}

// ------------------------------------------------------------------ draft sampling ----
// Draft sampling: a CTA takes kDsSpan logits of one request's draft row (two vocabulary
// chunks), staged in shared memory by one bulk copy (so no registers are held by loads in
// flight and a launch over 32 requests x 151,936 logits is one wave), and writes the two
// chunks' (max, sum) partials; the last CTA of the request merges them and draws.
constexpr int kDsPer = 2;
constexpr int kDsSpan = kDsPer * kVocabChunk;

// (max, sum) of this thread's entries t + 256 q of a staged chunk of n <= kVocabChunk, all
// 32 read from shared memory at once (no load latency per entry).
__device__ __forceinline__ void smem_ms(const float* xs, int n, float& m, float& s, bool& bad) {
  static_assert(kVocabChunk == 32 * kSampThreads, "32 entries per thread");
  float x[32];
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const int j = (int)threadIdx.x + kSampThreads * q;
    float v = j < n ? xs[j] : -INFINITY;
    if (isnan(v) || v == INFINITY) {
      bad = true;
      v = -INFINITY;
    }
    x[q] = v;
  }
  m = -INFINITY;
#pragma unroll
  for (int q = 0; q < 32; ++q) m = fmaxf(m, x[q]);
  s = 0.f;
  if (m != -INFINITY) {
    const float mb = m * kLog2e;
#pragma unroll
    for (int q = 0; q < 32; ++q) s += ex2(fmaf(x[q], kLog2e, -mb));
  }
}

__global__ void __launch_bounds__(kSampThreads) draft_sample_kernel(const SampleParams p) {
  pdl_wait();
  extern __shared__ float4 xs4[];   // [kDsSpan] logits of this CTA's span
  float* xs = reinterpret_cast<float*>(xs4);
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_flag;
  __shared__ double csum[64];
  __shared__ float s_M;
  const int cb = blockIdx.y, bl = blockIdx.x;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) {   // every CTA of the row returns: no ticket is touched
    if (cb == 0 && threadIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int i = p.draft_step[r];
  const int V = p.vocab;
  if (i < 0 || i >= p.k) {
    if (cb == 0 && threadIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const float* row = p.q_logits + ((size_t)r * p.k + i) * V;
  MS* part = reinterpret_cast<MS*>(p.part) + (size_t)r * p.nvch;
  const int v0 = cb * kDsSpan, n = min(V - v0, kDsSpan);

  // stage the span: one bulk copy when it is 16-byte aligned and sized, else plain loads
  const bool bulk = ((reinterpret_cast<uintptr_t>(row + v0) & 15u) == 0) && ((n & 3) == 0);
  if (bulk) {
    if (threadIdx.x == 0) {
      mbar_init(smem_u32(&bar), 1);
      fence_mbar_init();
    }
    __syncthreads();   // the barrier is initialised before the copy and before anyone polls it
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(smem_u32(&bar), (uint32_t)n * 4u);
      bulk_load(smem_u32(xs), row + v0, (uint32_t)n * 4u, smem_u32(&bar));
    }
    if (!mbar_wait(smem_u32(&bar), 0) && threadIdx.x == 0) set_error(p.err, S3R_ERR_TIMEOUT);
  } else {
    for (int j = threadIdx.x; j < n; j += kSampThreads) xs[j] = __ldg(row + v0 + j);
    __syncthreads();
  }

  bool bad = false;
#pragma unroll
  for (int h = 0; h < kDsPer; ++h) {
    const int c = cb * kDsPer + h;
    if (c >= p.nvch) break;
    float m, s;
    smem_ms(xs + h * kVocabChunk, min(n - h * kVocabChunk, kVocabChunk), m, s, bad);
    const MS tot = block_ms(m, s);
    if (threadIdx.x == 0) part[c] = tot;
    __syncthreads();   // block_ms's scratch is reused by the next chunk
  }
  if (bad) set_error(p.err, S3R_ERR_NONFINITE);
  if (!last_of(p.tickets + r, (int)gridDim.y, &s_flag)) return;

  if (threadIdx.x < 32) {
    const float M = merge_partials_warp(part, p.nvch, csum);
    if (threadIdx.x == 0) s_M = M;
  }
  __syncthreads();
  const float M = s_M;
  double Z = 0.0;
  for (int q = 0; q < p.nvch; ++q) Z += csum[q];
  const int L = p.seq_lens[r];
  const double u = philox_u(p.seed, (uint32_t)(L + i + 1), (uint32_t)r, 0u);
  const float Mb = M * kLog2e;
  // the chunk holding u * Z is staged in shared memory (the span's buffer, by a bulk copy
  // on the same barrier, whose phase 0 was the span's copy), then searched there
  uint32_t phase = 1;
  auto stage = [&](int c0, int cn) {
    if (bulk && (cn & 3) == 0) {
      if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(smem_u32(&bar), (uint32_t)cn * 4u);
        bulk_load(smem_u32(xs), row + c0, (uint32_t)cn * 4u, smem_u32(&bar));
      }
      if (!mbar_wait(smem_u32(&bar), phase & 1u) && threadIdx.x == 0) set_error(p.err, S3R_ERR_TIMEOUT);
      ++phase;
    } else {
      for (int j = threadIdx.x; j < cn; j += kSampThreads) xs[j] = __ldg(row + c0 + j);
      __syncthreads();
    }
  };
  auto wq = [&](float x) -> float { return (isnan(x) || x == INFINITY) ? 0.f : ex2(fmaf(x, kLog2e, -Mb)); };
  double mrg;
  const int tok = draw_staged(
      V, p.nvch, csum, u * Z, mrg, stage, [&](int v, int c0) { return wq(xs[v - c0]); },
      [&](int v) { return wq(row[v]); });
  if (threadIdx.x == 0) {
    p.draft_out[(size_t)r * p.k + i] = tok;
    if (p.margins) p.margins[(size_t)r * p.k + i] = Z > 0.0 ? (float)(mrg / Z) : 0.f;
  }
}

// ------------------------------------------------------- speculative sampling: pass 1 --
__global__ void __launch_bounds__(kSampThreads) spec_norm_kernel(const SampleParams p) {
  pdl_wait();
  __shared__ int s_flag;
  __shared__ float sM[2 * S3R_MAX_K + 1];
  __shared__ double sZ[2 * S3R_MAX_K + 1];
  const int bl = blockIdx.x, rw = blockIdx.y, c = blockIdx.z;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) {   // every CTA of the request returns
    if (rw == 0 && c == 0 && threadIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int k = p.k, V = p.vocab, nrows = 2 * k + 1;
  const float* row = (rw <= k) ? p.p_logits + ((size_t)r * (k + 1) + rw) * V
                               : p.q_logits + ((size_t)r * k + (rw - k - 1)) * V;
  MS* part = reinterpret_cast<MS*>(p.part) + (size_t)r * nrows * p.nvch;

  float m, s;
  bool bad = false;
  thread_ms(row, c * kVocabChunk, min(V, (c + 1) * kVocabChunk), m, s, bad);
  if (bad) set_error(p.err, S3R_ERR_NONFINITE);
  const MS tot = block_ms(m, s);
  if (threadIdx.x == 0) part[rw * p.nvch + c] = tot;
  if (!last_of(p.tickets + r, nrows * p.nvch, &s_flag)) return;

  // normalisers of every row: one warp per row, the row's chunk partials loaded in parallel
  __shared__ double s_cs[8][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int row = warp; row < nrows; row += kSampThreads / 32) {
    const float M = merge_partials_warp(part + row * p.nvch, p.nvch, s_cs[warp]);
    __syncwarp();
    double z = 0.0;
    for (int q = lane; q < p.nvch; q += 32) z += s_cs[warp][q];
    z = warp_sum_d(z);
    if (lane == 0) {
      sM[row] = M;
      sZ[row] = z;
    }
    __syncwarp();
  }
  __syncthreads();
  if (warp != 0) return;

  // the k accept tests at once (lane j tests draft j), then the first rejection by ballot
  const int L = p.seq_lens[r];
  const size_t pbase = (size_t)r * (k + 1) * V, qbase = (size_t)r * k * V;
  bool acc = false;
  int d = -1;
  double margin = 0.0;   // |u - p/q| of this lane's draft
  if (lane < k) {
    d = p.draft_tokens[(size_t)r * k + lane];
    if (d < 0 || d >= V) {
      set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    } else {
      const double pj = exp((double)p.p_logits[pbase + (size_t)lane * V + d] - (double)sM[lane]) / sZ[lane];
      const double qj = exp((double)p.q_logits[qbase + (size_t)lane * V + d] - (double)sM[k + 1 + lane]) /
                        sZ[k + 1 + lane];
      const double u = philox_u(p.seed, (uint32_t)(L + lane + 1), (uint32_t)r, 1u);
      acc = u * qj < pj;
      margin = qj > 0.0 ? fabs(u - pj / qj) : INFINITY;
    }
  }
  const unsigned rej = ~__ballot_sync(kFull, acc) & ((1u << k) - 1u);
  const int a = rej ? __ffs(rej) - 1 : k;      // drafts accepted before the first rejection
  if (lane < a) p.out_tokens[(size_t)r * (k + 1) + lane] = d;
  // the decided drafts' margins: the accepted ones and the first rejected one
  if (p.margins && lane < k && lane <= a) p.margins[(size_t)r * (k + 1) + lane] = (float)margin;
  if (lane != 0) return;
  const int type = a < k ? 0 : 1, jrow = a;
  SpecPlan* plan = reinterpret_cast<SpecPlan*>(p.part + p.plan_off) + r;
  SpecPlan pl;
  pl.type = type;
  pl.row = jrow;
  pl.a = a;
  pl.pad = 0;
  pl.mp = sM[jrow];
  pl.zp = sZ[jrow];
  pl.mq = (type == 0) ? sM[k + 1 + jrow] : 0.f;
  pl.zq = (type == 0) ? sZ[k + 1 + jrow] : 1.0;
  pl.u = philox_u(p.seed, (uint32_t)(L + jrow + 1), (uint32_t)r, 2u);
  *plan = pl;
  p.n_out[r] = a + 1;
}

// ------------------------------------------------------- speculative sampling: pass 2 --
__global__ void __launch_bounds__(kSampThreads) spec_draw_kernel(const SampleParams p) {
  pdl_wait();
  extern __shared__ float4 xs4[];   // the drawn chunk: p logits, then q logits
  float* xps = reinterpret_cast<float*>(xs4);
  float* xqs = xps + kVocabChunk;
  __shared__ int s_flag;
  __shared__ double csum[64];
  __shared__ int s_use_res;
  const int c = blockIdx.y, bl = blockIdx.x;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) return;   // reported by the first pass
  const int k = p.k, V = p.vocab;
  const SpecPlan pl = reinterpret_cast<const SpecPlan*>(p.part + p.plan_off)[r];
  const float* prow = p.p_logits + ((size_t)r * (k + 1) + pl.row) * V;
  const float* qrow = p.q_logits + ((size_t)r * k + (pl.type == 0 ? pl.row : 0)) * V;
  double2* part = reinterpret_cast<double2*>(p.part + p.draw_off) + (size_t)r * p.nvch;
  const bool resid = pl.type == 0;
  const float mpb = pl.mp * kLog2e, mqb = pl.mq * kLog2e;
  const float izp = (float)(1.0 / pl.zp), izq = (float)(1.0 / pl.zq);
  auto w_p = [&](int v) -> float {
    const float x = prow[v];
    return (isnan(x) || x == INFINITY) ? 0.f : ex2(fmaf(x, kLog2e, -mpb));
  };
  auto w_res = [&](int v) -> float {
    const float x = prow[v], y = qrow[v];
    const float pv = (isnan(x) || x == INFINITY) ? 0.f : ex2(fmaf(x, kLog2e, -mpb)) * izp;
    const float qv = (isnan(y) || y == INFINITY) ? 0.f : ex2(fmaf(y, kLog2e, -mqb)) * izq;
    return fmaxf(pv - qv, 0.f);
  };

  const int v0 = c * kVocabChunk, v1 = min(V, (c + 1) * kVocabChunk);
  float srf = 0.f, spf = 0.f;
  auto wp_x = [&](float x) -> float {
    return (isnan(x) || x == INFINITY) ? 0.f : ex2(fmaf(x, kLog2e, -mpb));
  };
  auto wres_xy = [&](float x, float y) -> float {
    const float pv = (isnan(x) || x == INFINITY) ? 0.f : ex2(fmaf(x, kLog2e, -mpb)) * izp;
    const float qv = (isnan(y) || y == INFINITY) ? 0.f : ex2(fmaf(y, kLog2e, -mqb)) * izq;
    return fmaxf(pv - qv, 0.f);
  };
  const bool vec = ((reinterpret_cast<uintptr_t>(prow + v0) & 15u) == 0) &&
                   ((reinterpret_cast<uintptr_t>(qrow + v0) & 15u) == 0) && (((v1 - v0) & 3) == 0);
  if (vec) {
    // 32 entries per thread as eight 16-byte loads of each row, all in flight at once
    float4 xp[8], xq[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int v = v0 + 4 * ((int)threadIdx.x + kSampThreads * j);
      xp[j] = v < v1 ? __ldg(reinterpret_cast<const float4*>(prow + v)) : make_float4(0.f, 0.f, 0.f, 0.f);
      xq[j] = (resid && v < v1) ? __ldg(reinterpret_cast<const float4*>(qrow + v))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int v = v0 + 4 * ((int)threadIdx.x + kSampThreads * j);
      if (v < v1) {
        spf += wp_x(xp[j].x) + wp_x(xp[j].y) + wp_x(xp[j].z) + wp_x(xp[j].w);
        if (resid)
          srf += wres_xy(xp[j].x, xq[j].x) + wres_xy(xp[j].y, xq[j].y) +
                 wres_xy(xp[j].z, xq[j].z) + wres_xy(xp[j].w, xq[j].w);
      }
    }
  } else {
    for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
      spf += w_p(v);
      if (resid) srf += w_res(v);
    }
  }
  double sr = srf, sp = spf;
  sp = block_sum_d(sp);
  sr = block_sum_d(sr);
  if (threadIdx.x == 0) part[c] = make_double2(sr, sp);
  if (!last_of(p.tickets + r, p.nvch, &s_flag)) return;

  if (threadIdx.x < 32) {
    // chunk sums loaded by the lanes at once; the residual mass decides which row is drawn
    const int lane = threadIdx.x;
    double2 pq[2] = {make_double2(0.0, 0.0), make_double2(0.0, 0.0)};
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (lane + 32 * h < p.nvch) pq[h] = __ldcg(&part[lane + 32 * h]);
    const double zr = warp_sum_d(pq[0].x + pq[1].x);
    const int use_res = resid && zr > 0.0;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (lane + 32 * h < p.nvch) csum[lane + 32 * h] = use_res ? pq[h].x : pq[h].y;
    if (lane == 0) s_use_res = use_res;
  }
  __syncthreads();
  double Z = 0.0;
  for (int q = 0; q < p.nvch; ++q) Z += csum[q];
  const double target = pl.u * Z;
  const bool use_res = s_use_res != 0;
  // the drawn chunk of the p row (and the q row for a residual) staged in shared memory by
  // bulk copies (or plain loads when unaligned), then searched there
  __shared__ __align__(8) uint64_t bar;
  uint32_t phase = 0;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto stage = [&](int c0, int cn) {
    const bool v4 = ((reinterpret_cast<uintptr_t>(prow + c0) & 15u) == 0) &&
                    ((reinterpret_cast<uintptr_t>(qrow + c0) & 15u) == 0) && ((cn & 3) == 0);
    if (v4) {
      if (threadIdx.x == 0) {
        const uint32_t bytes = (uint32_t)cn * 4u;
        mbar_arrive_expect_tx(smem_u32(&bar), use_res ? 2u * bytes : bytes);
        bulk_load(smem_u32(xps), prow + c0, bytes, smem_u32(&bar));
        if (use_res) bulk_load(smem_u32(xqs), qrow + c0, bytes, smem_u32(&bar));
      }
      if (!mbar_wait(smem_u32(&bar), phase & 1u) && threadIdx.x == 0) set_error(p.err, S3R_ERR_TIMEOUT);
      ++phase;
      return;
    } else {
      for (int j = threadIdx.x; j < cn; j += kSampThreads) {
        xps[j] = __ldg(prow + c0 + j);
        if (use_res) xqs[j] = __ldg(qrow + c0 + j);
      }
    }
    __syncthreads();
  };
  int tok;
  double mrg;
  if (use_res)
    tok = draw_staged(V, p.nvch, csum, target, mrg, stage,
                      [&](int v, int c0) { return wres_xy(xps[v - c0], xqs[v - c0]); }, w_res);
  else
    tok = draw_staged(V, p.nvch, csum, target, mrg, stage,
                      [&](int v, int c0) { return wp_x(xps[v - c0]); }, w_p);
  if (threadIdx.x == 0) {
    p.out_tokens[(size_t)r * (k + 1) + pl.a] = tok;
    // the draw's margin follows the decided drafts' margins
    if (p.margins) p.margins[(size_t)r * (k + 1) + (pl.a < k ? pl.a + 1 : k)] = Z > 0.0 ? (float)(mrg / Z) : 0.f;
  }
}

// ------------------------------------------------------------ greedy (temperature 0) ----
// Argmax of logit rows, ties to the lowest token id, NaN counted as -inf (and flagged).
// mode 0: one row per request, the draft row of its step -> draft_tokens.
// mode 1: the k+1 target rows of each request -> drafts kept while they equal the target
//         argmax, the first mismatch replaced by it, the bonus token when all k agree.
// Grid (request, row, vocabulary chunk); the last CTA of a request merges and decides.
struct ArgMax {
  float v;
  int i;
};
static_assert(sizeof(ArgMax) <= sizeof(MS), "argmax partials reuse the (m, s) partial slots");
__device__ __forceinline__ ArgMax better(ArgMax a, ArgMax b) {
  return (b.v > a.v || (b.v == a.v && b.i < a.i)) ? b : a;
}
__device__ __forceinline__ ArgMax warp_argmax(ArgMax a) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    ArgMax b;
    b.v = __shfl_xor_sync(kFull, a.v, o);
    b.i = __shfl_xor_sync(kFull, a.i, o);
    a = better(a, b);
  }
  return a;
}

__global__ void __launch_bounds__(kSampThreads) argmax_kernel(const SampleParams p, int mode) {
  pdl_wait();
  __shared__ int s_flag;
  __shared__ ArgMax s_w[kSampThreads / 32];
  __shared__ ArgMax s_part[(S3R_MAX_K + 1) * 64];
  __shared__ ArgMax s_row[S3R_MAX_K + 1];
  const int bl = blockIdx.x, j = blockIdx.y, c = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) {   // every CTA of the request returns
    if (j == 0 && c == 0 && threadIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int k = p.k, V = p.vocab;
  const int nrows = mode == 0 ? 1 : k + 1;
  const float* row;
  int i = 0;
  if (mode == 0) {
    i = p.draft_step[r];
    if (i < 0 || i >= k) {
      if (c == 0 && threadIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
      return;
    }
    row = p.q_logits + ((size_t)r * k + i) * V;
  } else {
    row = p.p_logits + ((size_t)r * (k + 1) + j) * V;
  }
  const int v0 = c * kVocabChunk, v1 = min(V, (c + 1) * kVocabChunk);
  ArgMax best{-INFINITY, INT_MAX};
  bool bad = false;
#pragma unroll 8
  for (int q = 0; q < kVocabChunk / kSampThreads; ++q) {
    const int v = v0 + (int)threadIdx.x + kSampThreads * q;
    if (v < v1) {
      float x = __ldg(row + v);
      if (isnan(x)) {
        bad = true;
        x = -INFINITY;
      }
      best = better(best, ArgMax{x, v});
    }
  }
  if (bad) set_error(p.err, S3R_ERR_NONFINITE);
  best = warp_argmax(best);
  if (lane == 0) s_w[warp] = best;
  __syncthreads();
  ArgMax* part = reinterpret_cast<ArgMax*>(p.part) + (size_t)r * nrows * p.nvch;
  if (threadIdx.x == 0) {
    ArgMax b = s_w[0];
    for (int w = 1; w < kSampThreads / 32; ++w) b = better(b, s_w[w]);
    part[j * p.nvch + c] = b;
  }
  if (!last_of(p.tickets + r, nrows * p.nvch, &s_flag)) return;

  // every (row, chunk) partial at once, then one warp per row
  for (int t = threadIdx.x; t < nrows * p.nvch; t += blockDim.x) {
    ArgMax a;
    a.v = __ldcg(&part[t].v);
    a.i = __ldcg(&part[t].i);
    s_part[t] = a;
  }
  __syncthreads();
  for (int rr = warp; rr < nrows; rr += kSampThreads / 32) {
    ArgMax b{-INFINITY, INT_MAX};
    for (int q = lane; q < p.nvch; q += 32) b = better(b, s_part[rr * p.nvch + q]);
    b = warp_argmax(b);
    if (lane == 0) s_row[rr] = b;
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  // a row of only -inf has no maximum above -inf: its argmax is token 0 (lowest id)
  auto tok = [&](int rr) { return s_row[rr].i == INT_MAX ? 0 : s_row[rr].i; };
  if (mode == 0) {
    p.draft_out[(size_t)r * k + i] = tok(0);
    return;
  }
  int a = 0;
  while (a < k) {
    const int d = p.draft_tokens[(size_t)r * k + a];
    if (d != tok(a)) break;
    ++a;
  }
  for (int t = 0; t <= a; ++t) p.out_tokens[(size_t)r * (k + 1) + t] = tok(t);
  p.n_out[r] = a + 1;
}

int launch_argmax(const SampleParams& p, int batch, int mode, cudaStream_t stream) {
  dim3 grid(batch, mode == 0 ? 1 : p.k + 1, p.nvch);
  launch_pdl(argmax_kernel, grid, kSampThreads, 0, stream, p, mode);
  return cuda_status(cudaGetLastError(), __func__);
}

// ------------------------------------------------------------------------- commit ----
__global__ void commit_kernel(const int32_t* req_ids, int batch, int k, const int32_t* n_out,
                              int32_t* seq_lens, long long* stats) {
  pdl_wait();
  const int bl = blockIdx.x * blockDim.x + threadIdx.x;
  if (bl >= batch) return;
  const int r = req_ids ? req_ids[bl] : bl;
  const int n = n_out[r];
  seq_lens[r] += n;
  if (stats) {
    atomicAdd(reinterpret_cast<unsigned long long*>(&stats[0]), (unsigned long long)n);
    atomicAdd(reinterpret_cast<unsigned long long*>(&stats[1]), 1ull);
    for (int j = 0; j < k && j < n; ++j) {
      atomicAdd(reinterpret_cast<unsigned long long*>(&stats[2 + S3R_MAX_K + j]), 1ull);
      if (j < n - 1) atomicAdd(reinterpret_cast<unsigned long long*>(&stats[2 + j]), 1ull);
    }
  }
}

__global__ void philox_kernel(uint64_t seed, int stream_id, const int32_t* request,
                              const int32_t* position, int64_t n, uint32_t* words, float* u) {
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  uint32_t c[4] = {(uint32_t)position[i], (uint32_t)request[i], (uint32_t)stream_id, 0u};
  philox4x32_10(c, (uint32_t)seed, (uint32_t)(seed >> 32));
  if (words) {
    words[4 * i + 0] = c[0];
    words[4 * i + 1] = c[1];
    words[4 * i + 2] = c[2];
    words[4 * i + 3] = c[3];
  }
  if (u) u[i] = (float)(c[0] >> 8) * (1.0f / 16777216.0f);
}

// ------------------------------------------------------------------------ launchers ----
int launch_draft_sample(const SampleParams& p, int batch, cudaStream_t stream) {
  constexpr int smem = kDsSpan * 4;
  static std::atomic<uint64_t> attr_done{0};
  if (cuda_status(ensure_smem_attr(draft_sample_kernel, smem, attr_done), "cudaFuncSetAttribute") != S3R_OK)
    return S3R_ERR_CUDA;
  dim3 grid(batch, (p.vocab + kDsSpan - 1) / kDsSpan);
  launch_pdl(draft_sample_kernel, grid, kSampThreads, smem, stream, p);
  return cuda_status(cudaGetLastError(), __func__);
}

int launch_spec_sample(const SampleParams& p, int batch, cudaStream_t stream, int* launches) {
  dim3 g1(batch, 2 * p.k + 1, p.nvch);
  launch_pdl(spec_norm_kernel, g1, kSampThreads, 0, stream, p);
  if (cuda_status(cudaGetLastError(), __func__) != S3R_OK) return S3R_ERR_CUDA;
  constexpr int smem2 = 2 * kVocabChunk * 4;
  static std::atomic<uint64_t> attr_done{0};
  if (cuda_status(ensure_smem_attr(spec_draw_kernel, smem2, attr_done), "cudaFuncSetAttribute") != S3R_OK)
    return S3R_ERR_CUDA;
  dim3 g2(batch, p.nvch);
  launch_pdl(spec_draw_kernel, g2, kSampThreads, smem2, stream, p);
  *launches = 2;
  return cuda_status(cudaGetLastError(), __func__);
}

size_t sample_partial_bytes(int num_requests, int k, int vocab) {
  const size_t nvch = (size_t)((vocab + kVocabChunk - 1) / kVocabChunk);
  const size_t a = align_up((size_t)num_requests * (2 * k + 1) * nvch * sizeof(MS), 256);
  const size_t b = align_up((size_t)num_requests * sizeof(SpecPlan), 256);
  const size_t c = align_up((size_t)num_requests * nvch * sizeof(double2), 256);
  return a + b + c;
}

void spec_offsets(int num_requests, int k, int vocab, size_t* plan_off, size_t* draw_off) {
  const size_t nvch = (size_t)((vocab + kVocabChunk - 1) / kVocabChunk);
  *plan_off = align_up((size_t)num_requests * (2 * k + 1) * nvch * sizeof(MS), 256);
  *draw_off = *plan_off + align_up((size_t)num_requests * sizeof(SpecPlan), 256);
}

int launch_commit(const int32_t* req_ids, int batch, int k, const int32_t* n_out,
                  int32_t* seq_lens, int64_t* stats, cudaStream_t stream) {
  launch_pdl(commit_kernel, (batch + 255) / 256, 256, 0, stream, req_ids, batch, k, n_out, seq_lens,
                                                        reinterpret_cast<long long*>(stats));
  return cuda_status(cudaGetLastError(), __func__);
}

int launch_philox(uint64_t seed, int stream_id, const int32_t* request, const int32_t* position,
                  int64_t n, uint32_t* words, float* u, cudaStream_t stream) {
  launch_pdl(philox_kernel, (unsigned)((n + 255) / 256), 256, 0, stream, seed, stream_id, request, position,
                                                                 n, words, u);
  return cuda_status(cudaGetLastError(), __func__);
}

}  // namespace s3r
