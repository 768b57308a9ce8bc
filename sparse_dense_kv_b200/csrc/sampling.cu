// Draft-token sampling, exact speculative sampling, round commit and Philox uniforms.
//
// What they compute ([News] Interpretation and [Explainer] Jargon, exact speculative
// sampling: accept a draft or draw from the residual distribution so that emitted tokens
// follow the dense policy): softmax normalisers of the draft / target rows, the accept
// tests u * q(d) < p(d), and inverse-CDF draws from q, from max(0, p - q) or from p.
//
// The vocabulary is split into chunks of 8192 entries. A pass over (chunk, row, request)
// produces (max, sum exp(x - max)) per chunk with fp32 exponentials and fp64 sums; the last
// CTA of a request merges the chunks (ticket, no spinning) and decides. For a draw the pass
// also writes the sums of the chunk's eight sub-blocks of 1024 entries, so the last CTA
// finds the chunk and then the sub-block holding u * Z from sums alone, and reads and
// searches only that sub-block's 1024 logits (one 16-byte load per thread, a block-wide
// prefix sum in fp64).
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

// ----------------------------------------------------------------- sub-block draws ----
constexpr int kSub = 1024;                     // entries per sub-block sum
constexpr int kSubPer = kVocabChunk / kSub;    // sub-blocks per vocabulary chunk (8)
static_assert(kSub == 4 * kSampThreads, "one 16-byte load of a sub-block per thread");

// Sum over the block of each thread's kSubPer values; out[0..kSubPer) valid after return
// in every thread (fp32 warp sums, fp32 across the warps).
__device__ __forceinline__ void block_sum_sub(float (&v)[kSubPer], float* out) {
  __shared__ float sw[kSampThreads / 32][kSubPer];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int b = 0; b < kSubPer; ++b) {
    float x = v[b];
#pragma unroll
    for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    if (lane == 0) sw[warp][b] = x;
  }
  __syncthreads();
  if (threadIdx.x < kSubPer) {
    float t = 0.f;
    for (int w = 0; w < kSampThreads / 32; ++w) t += sw[w][threadIdx.x];
    out[threadIdx.x] = t;
  }
  __syncthreads();
}

// The draw of the last CTA of a request: target = u * Z on the weights' common scale, the
// chunk sums csum[0..nvch) (that scale), sub(c, b) the sum of sub-block b of chunk c (that
// scale). Thread 0 walks the chunk sums, then the chosen chunk's sub-block sums; then every
// thread takes 4 consecutive entries of the sub-block (weight4(v0, w) fills w[0..3] on the
// common scale, 0 past the vocabulary), and a block-wide fp64 prefix sum finds the smallest v
// with target < C_v. `mrg` receives the target's distance to the nearer edge of v's cell
// (0 where rounding carried the target past the sub-block: its last non-zero entry is taken).
template <class Sub, class W4>
__device__ int subblock_draw(int V, int nvch, const double* csum, double target, double& mrg, Sub sub,
                             W4 weight4) {
  __shared__ int s_c, s_b, s_tok, s_last;
  __shared__ double s_base, s_mrg;
  __shared__ double s_wt[kSampThreads / 32];
  if (threadIdx.x == 0) {
    double cum = 0.0;
    int c = -1, lastc = -1;
    for (int i = 0; i < nvch; ++i) {
      if (csum[i] > 0.0) lastc = i;
      if (c < 0 && target < cum + csum[i]) c = i;
      if (c < 0) cum += csum[i];
    }
    int b = -1;
    if (c < 0) {                      // rounding past the last chunk: its last sub-block
      c = lastc < 0 ? 0 : lastc;
      cum = 0.0;
      for (int i = 0; i < c; ++i) cum += csum[i];
      for (int j = 0; j < kSubPer; ++j)
        if (sub(c, j) > 0.0) b = j;
      for (int j = 0; j < b; ++j) cum += sub(c, j);
    } else {
      int lastb = 0;
      for (int j = 0; j < kSubPer && b < 0; ++j) {
        const double sj = sub(c, j);
        if (sj > 0.0) lastb = j;
        if (target < cum + sj) b = j;
        else cum += sj;
      }
      if (b < 0) {                    // rounding past the chunk's last sub-block
        b = lastb;
        cum = 0.0;
        for (int i = 0; i < c; ++i) cum += csum[i];
        for (int j = 0; j < b; ++j) cum += sub(c, j);
      }
    }
    s_c = c;
    s_b = b < 0 ? 0 : b;
    s_base = cum;
    s_tok = INT_MAX;
    s_last = -1;
    s_mrg = 0.0;
  }
  __syncthreads();
  const int v0 = s_c * kVocabChunk + s_b * kSub + 4 * (int)threadIdx.x;
  double w[4];
  weight4(v0, w);
  const double mine = (w[0] + w[1]) + (w[2] + w[3]);
  // block exclusive prefix of the threads' sums (fp64)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_wt[warp] = incl;
  __syncthreads();
  double before = s_base;
  for (int q = 0; q < warp; ++q) before += s_wt[q];
  double c0 = before + incl - mine;
  int last_nz = -1;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (w[e] > 0.0) {
      last_nz = v0 + e;
      if (target >= c0 && target < c0 + w[e]) {   // cells are disjoint: one entry at most
        s_tok = v0 + e;
        s_mrg = fmin(target - c0, c0 + w[e] - target);
      }
    }
    c0 += w[e];
  }
  if (last_nz >= 0) atomicMax(&s_last, last_nz);
  __syncthreads();
  int tok = s_tok;
  mrg = s_mrg;
  if (tok == INT_MAX) {               // rounding past the sub-block: its last non-zero entry
    tok = s_last >= 0 ? s_last : min(v0, V - 1);
    mrg = 0.0;
  }
  __syncthreads();
  return tok;
}

// ------------------------------------------------------------------ draft sampling ----
// Draft sampling: a CTA takes one vocabulary chunk (8192 logits) of one request's draft row,
// eight 16-byte loads per thread all in flight at once (load j of thread t holds entries
// 1024 j + 4 t .. + 3, so it lies in sub-block j), and writes the chunk's (max, sum) partial
// and its sub-block sums; the last CTA of the request merges them and draws from the one
// sub-block that holds u * Z. At most 51 registers a thread, so five CTAs fit on an SM and a
// launch over 32 requests x 151,936 logits (608 CTAs) is one wave.
constexpr int kDsMinBlocks = 5;

__global__ void __launch_bounds__(kSampThreads, kDsMinBlocks) draft_sample_kernel(const SampleParams p) {
  pdl_wait();
  __shared__ int s_flag;
  __shared__ double csum[64];
  __shared__ float s_mc[64];        // chunk maxima
  __shared__ float s_red[kSampThreads / 32];
  __shared__ float s_sub[kSubPer];
  __shared__ float s_subs[64 * kSubPer];
  __shared__ float s_M;
  const int c = blockIdx.y, bl = blockIdx.x;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) {   // every CTA of the row returns: no ticket is touched
    if (c == 0 && threadIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int i = p.draft_step[r];
  const int L = p.seq_lens[r];      // read now: both loads in flight together
  const int V = p.vocab;
  if (i < 0 || i >= p.k) {
    if (c == 0 && threadIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const float* row = p.q_logits + ((size_t)r * p.k + i) * V;
  MS* part = reinterpret_cast<MS*>(p.part) + (size_t)r * p.nvch;
  float* subs = reinterpret_cast<float*>(p.part + p.sub_off) + (size_t)r * p.nvch * kSubPer;
  const int v0 = c * kVocabChunk, v1 = min(V, v0 + kVocabChunk);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  float4 x[kSubPer];
  const bool vec = ((reinterpret_cast<uintptr_t>(row + v0) & 15u) == 0) && (((v1 - v0) & 3) == 0);
#pragma unroll
  for (int j = 0; j < kSubPer; ++j) {
    const int v = v0 + kSub * j + 4 * (int)threadIdx.x;
    if (vec) {
      x[j] = v < v1 ? __ldg(reinterpret_cast<const float4*>(row + v))
                    : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    } else {
      x[j].x = v < v1 ? __ldg(row + v) : -INFINITY;
      x[j].y = v + 1 < v1 ? __ldg(row + v + 1) : -INFINITY;
      x[j].z = v + 2 < v1 ? __ldg(row + v + 2) : -INFINITY;
      x[j].w = v + 3 < v1 ? __ldg(row + v + 3) : -INFINITY;
    }
  }
  bool bad = false;
  float m = -INFINITY;
  auto clean = [&](float& v) {
    if (isnan(v) || v == INFINITY) {
      bad = true;
      v = -INFINITY;
    }
  };
#pragma unroll
  for (int j = 0; j < kSubPer; ++j) {
    clean(x[j].x);
    clean(x[j].y);
    clean(x[j].z);
    clean(x[j].w);
    m = fmaxf(fmaxf(m, fmaxf(x[j].x, x[j].y)), fmaxf(x[j].z, x[j].w));
  }
  if (bad) set_error(p.err, S3R_ERR_NONFINITE);
  m = warp_max(m);
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  float Mc = s_red[0];
  for (int w = 1; w < kSampThreads / 32; ++w) Mc = fmaxf(Mc, s_red[w]);
  float sub[kSubPer];
  const float mb = Mc * kLog2e;
#pragma unroll
  for (int j = 0; j < kSubPer; ++j)
    sub[j] = Mc == -INFINITY ? 0.f
                             : (ex2(fmaf(x[j].x, kLog2e, -mb)) + ex2(fmaf(x[j].y, kLog2e, -mb))) +
                                   (ex2(fmaf(x[j].z, kLog2e, -mb)) + ex2(fmaf(x[j].w, kLog2e, -mb)));
  block_sum_sub(sub, s_sub);
  if (threadIdx.x < kSubPer) subs[(size_t)c * kSubPer + threadIdx.x] = s_sub[threadIdx.x];
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int b = 0; b < kSubPer; ++b) t += (double)s_sub[b];
    MS tot;
    tot.m = Mc;
    tot.pad = 0.f;
    tot.s = t;
    part[c] = tot;
  }
  if (!last_of(p.tickets + r, (int)gridDim.y, &s_flag)) return;

  // the last CTA: chunk maxima and weights on the common scale, every sub-block sum
  if (threadIdx.x < 32) {
    const float M = merge_partials_warp(part, p.nvch, csum);
    if (threadIdx.x == 0) s_M = M;
    for (int q = threadIdx.x; q < p.nvch; q += 32) s_mc[q] = __ldcg(&part[q].m);
  }
  for (int t = threadIdx.x; t < p.nvch * kSubPer; t += kSampThreads) s_subs[t] = __ldcg(subs + t);
  __syncthreads();
  const float M = s_M;
  double Z = 0.0;
  for (int q = 0; q < p.nvch; ++q) Z += csum[q];
  const double u = philox_u(p.seed, (uint32_t)(L + i + 1), (uint32_t)r, 0u);
  auto scale = [&](int cc) -> double {   // chunk cc's weights -> the common scale
    return s_mc[cc] == -INFINITY ? 0.0 : (double)exp2f((s_mc[cc] - M) * kLog2e);
  };
  double mrg;
  const int tok = subblock_draw(
      V, p.nvch, csum, u * Z, mrg, [&](int cc, int b) { return (double)s_subs[cc * kSubPer + b] * scale(cc); },
      [&](int vw, double (&w)[4]) {
        const int cc = vw / kVocabChunk;
        const float mbc = s_mc[cc] * kLog2e;
        const double f = scale(cc);
        float xv[4];
        if (vw + 3 < V && ((reinterpret_cast<uintptr_t>(row + vw) & 15u) == 0)) {
          const float4 t = __ldg(reinterpret_cast<const float4*>(row + vw));
          xv[0] = t.x; xv[1] = t.y; xv[2] = t.z; xv[3] = t.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) xv[e] = vw + e < V ? __ldg(row + vw + e) : -INFINITY;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float xe = (isnan(xv[e]) || xv[e] == INFINITY) ? -INFINITY : xv[e];
          w[e] = (s_mc[cc] == -INFINITY) ? 0.0 : (double)ex2(fmaf(xe, kLog2e, -mbc)) * f;
        }
      });
  if (threadIdx.x == 0) {
    p.draft_out[(size_t)r * p.k + i] = tok;
    if (p.margins) p.margins[(size_t)r * p.k + i] = Z > 0.0 ? (float)(mrg / Z) : 0.f;
    if (p.q_norm) {
      s3r_row_norm nm;
      nm.max = M;
      nm.reserved = 0.f;
      nm.sum = Z;
      p.q_norm[(size_t)r * p.k + i] = nm;
    }
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
  // rows 0..k: p, rows k+1..2k: q; with the draft rows' normalisers given, only the p rows
  // are streamed (the grid's second dimension is k + 1)
  const int nstream = p.q_norm ? k + 1 : nrows;
  const float* row = (rw <= k) ? p.p_logits + ((size_t)r * (k + 1) + rw) * V
                               : p.q_logits + ((size_t)r * k + (rw - k - 1)) * V;
  MS* part = reinterpret_cast<MS*>(p.part) + (size_t)r * nrows * p.nvch;

  float m, s;
  bool bad = false;
  thread_ms(row, c * kVocabChunk, min(V, (c + 1) * kVocabChunk), m, s, bad);
  if (bad) set_error(p.err, S3R_ERR_NONFINITE);
  const MS tot = block_ms(m, s);
  if (threadIdx.x == 0) part[rw * p.nvch + c] = tot;
  if (!last_of(p.tickets + r, nstream * p.nvch, &s_flag)) return;

  // normalisers of every row: one warp per streamed row, the row's chunk partials loaded in
  // parallel; the q rows' from q_norm when given
  __shared__ double s_cs[8][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (p.q_norm && (int)threadIdx.x < k) {
    const s3r_row_norm nm = p.q_norm[(size_t)r * k + threadIdx.x];
    sM[k + 1 + threadIdx.x] = nm.max;
    sZ[k + 1 + threadIdx.x] = nm.sum;
  }
  for (int row = warp; row < nstream; row += kSampThreads / 32) {
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
// The drawn row's chunk sums of the residual max(0, p - q) and of p, with the sums of their
// sub-blocks; the last CTA draws from the residual (or from p if its mass is zero).
__global__ void __launch_bounds__(kSampThreads, kDsMinBlocks) spec_draw_kernel(const SampleParams p) {
  pdl_wait();
  __shared__ int s_flag;
  __shared__ double csum[64];
  __shared__ int s_use_res;
  __shared__ float s_subr[kSubPer], s_subp[kSubPer];
  __shared__ float s_subs[64 * kSubPer];
  const int c = blockIdx.y, bl = blockIdx.x;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) return;   // reported by the first pass
  const int k = p.k, V = p.vocab;
  const SpecPlan pl = reinterpret_cast<const SpecPlan*>(p.part + p.plan_off)[r];
  const float* prow = p.p_logits + ((size_t)r * (k + 1) + pl.row) * V;
  const float* qrow = p.q_logits + ((size_t)r * k + (pl.type == 0 ? pl.row : 0)) * V;
  double2* part = reinterpret_cast<double2*>(p.part + p.draw_off) + (size_t)r * p.nvch;
  float* subs = reinterpret_cast<float*>(p.part + p.sub_off) + (size_t)r * p.nvch * 2 * kSubPer;
  const bool resid = pl.type == 0;
  const float mpb = pl.mp * kLog2e, mqb = pl.mq * kLog2e;
  const float izp = (float)(1.0 / pl.zp), izq = (float)(1.0 / pl.zq);
  auto wp_x = [&](float x) -> float {
    return (isnan(x) || x == INFINITY) ? 0.f : ex2(fmaf(x, kLog2e, -mpb));
  };
  auto wres_xy = [&](float x, float y) -> float {
    const float pv = (isnan(x) || x == INFINITY) ? 0.f : ex2(fmaf(x, kLog2e, -mpb)) * izp;
    const float qv = (isnan(y) || y == INFINITY) ? 0.f : ex2(fmaf(y, kLog2e, -mqb)) * izq;
    return fmaxf(pv - qv, 0.f);
  };

  const int v0 = c * kVocabChunk, v1 = min(V, (c + 1) * kVocabChunk);
  float subr[kSubPer], subp[kSubPer];
#pragma unroll
  for (int b = 0; b < kSubPer; ++b) subr[b] = subp[b] = 0.f;
  const bool vec = ((reinterpret_cast<uintptr_t>(prow + v0) & 15u) == 0) &&
                   ((reinterpret_cast<uintptr_t>(qrow + v0) & 15u) == 0) && (((v1 - v0) & 3) == 0);
  if (vec) {
    // 32 entries per thread as eight 16-byte loads of each row, four of each in flight at a
    // time (the register budget of five CTAs per SM); load j of every thread covers sub-block j
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float4 xp[4], xq[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int v = v0 + 4 * ((int)threadIdx.x + kSampThreads * (4 * h + jj));
        xp[jj] = v < v1 ? __ldg(reinterpret_cast<const float4*>(prow + v)) : make_float4(0.f, 0.f, 0.f, 0.f);
        xq[jj] = (resid && v < v1) ? __ldg(reinterpret_cast<const float4*>(qrow + v))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = 4 * h + jj;
        const int v = v0 + 4 * ((int)threadIdx.x + kSampThreads * j);
        if (v < v1) {
          subp[j] = wp_x(xp[jj].x) + wp_x(xp[jj].y) + wp_x(xp[jj].z) + wp_x(xp[jj].w);
          if (resid)
            subr[j] = wres_xy(xp[jj].x, xq[jj].x) + wres_xy(xp[jj].y, xq[jj].y) +
                      wres_xy(xp[jj].z, xq[jj].z) + wres_xy(xp[jj].w, xq[jj].w);
        }
      }
    }
  } else {
    for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
      const int b = (v - v0) / kSub;
      const float x = prow[v];
      subp[b] += wp_x(x);
      if (resid) subr[b] += wres_xy(x, qrow[v]);
    }
  }
  block_sum_sub(subr, s_subr);
  block_sum_sub(subp, s_subp);
  if (threadIdx.x < kSubPer) {
    subs[((size_t)c * 2) * kSubPer + threadIdx.x] = s_subr[threadIdx.x];
    subs[((size_t)c * 2 + 1) * kSubPer + threadIdx.x] = s_subp[threadIdx.x];
  }
  if (threadIdx.x == 0) {
    double sr = 0.0, sp = 0.0;
    for (int b = 0; b < kSubPer; ++b) {
      sr += (double)s_subr[b];
      sp += (double)s_subp[b];
    }
    part[c] = make_double2(sr, sp);
  }
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
  const bool use_res = s_use_res != 0;
  for (int t = threadIdx.x; t < p.nvch * kSubPer; t += kSampThreads) {
    const int cc = t / kSubPer, b = t - cc * kSubPer;
    s_subs[t] = __ldcg(subs + ((size_t)cc * 2 + (use_res ? 0 : 1)) * kSubPer + b);
  }
  __syncthreads();
  double Z = 0.0;
  for (int q = 0; q < p.nvch; ++q) Z += csum[q];
  const double target = pl.u * Z;
  double mrg;
  const int tok = subblock_draw(
      V, p.nvch, csum, target, mrg, [&](int cc, int b) { return (double)s_subs[cc * kSubPer + b]; },
      [&](int vw, double (&w)[4]) {
        float xp[4], xq[4];
        const bool al = vw + 3 < V && ((reinterpret_cast<uintptr_t>(prow + vw) & 15u) == 0) &&
                        ((reinterpret_cast<uintptr_t>(qrow + vw) & 15u) == 0);
        if (al) {
          const float4 a = __ldg(reinterpret_cast<const float4*>(prow + vw));
          xp[0] = a.x; xp[1] = a.y; xp[2] = a.z; xp[3] = a.w;
          if (use_res) {
            const float4 b = __ldg(reinterpret_cast<const float4*>(qrow + vw));
            xq[0] = b.x; xq[1] = b.y; xq[2] = b.z; xq[3] = b.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            xp[e] = vw + e < V ? __ldg(prow + vw + e) : -INFINITY;
            xq[e] = (use_res && vw + e < V) ? __ldg(qrow + vw + e) : -INFINITY;
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] = vw + e >= V ? 0.0 : (double)(use_res ? wres_xy(xp[e], xq[e]) : wp_x(xp[e]));
      });
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
__global__ void commit_kernel(const int32_t* req_ids, int batch, int num_requests, int k,
                              const int32_t* n_out, int32_t* seq_lens, long long* stats) {
  pdl_wait();
  const int bl = blockIdx.x * blockDim.x + threadIdx.x;
  if (bl >= batch) return;
  const int r = req_ids ? req_ids[bl] : bl;
  if (r < 0 || r >= num_requests) return;   // skipped (the commit has no error word)
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
  dim3 grid(batch, p.nvch);
  launch_pdl(draft_sample_kernel, grid, kSampThreads, 0, stream, p);
  return cuda_status(cudaGetLastError(), __func__);
}

int launch_spec_sample(const SampleParams& p, int batch, cudaStream_t stream, int* launches) {
  dim3 g1(batch, p.q_norm ? p.k + 1 : 2 * p.k + 1, p.nvch);
  launch_pdl(spec_norm_kernel, g1, kSampThreads, 0, stream, p);
  if (cuda_status(cudaGetLastError(), __func__) != S3R_OK) return S3R_ERR_CUDA;
  dim3 g2(batch, p.nvch);
  launch_pdl(spec_draw_kernel, g2, kSampThreads, 0, stream, p);
  *launches = 2;
  return cuda_status(cudaGetLastError(), __func__);
}

// Speculative sampling's workspace: normaliser partials [NR][2k+1][nvch], plans [NR], draw
// partials [NR][nvch] (double2), draw sub-block sums [NR][nvch][2][kSubPer] (fp32).
// Draft sampling's: partials [NR][nvch], then sub-block sums [NR][nvch][kSubPer].
size_t sample_partial_bytes(int num_requests, int k, int vocab) {
  const size_t nvch = (size_t)((vocab + kVocabChunk - 1) / kVocabChunk);
  const size_t a = align_up((size_t)num_requests * (2 * k + 1) * nvch * sizeof(MS), 256);
  const size_t b = align_up((size_t)num_requests * sizeof(SpecPlan), 256);
  const size_t c = align_up((size_t)num_requests * nvch * sizeof(double2), 256);
  const size_t d = align_up((size_t)num_requests * nvch * 2 * kSubPer * sizeof(float), 256);
  const size_t draft = draft_sub_offset(num_requests, vocab) +
                       align_up((size_t)num_requests * nvch * kSubPer * sizeof(float), 256);
  return a + b + c + d > draft ? a + b + c + d : draft;
}

void spec_offsets(int num_requests, int k, int vocab, size_t* plan_off, size_t* draw_off, size_t* sub_off) {
  const size_t nvch = (size_t)((vocab + kVocabChunk - 1) / kVocabChunk);
  *plan_off = align_up((size_t)num_requests * (2 * k + 1) * nvch * sizeof(MS), 256);
  *draw_off = *plan_off + align_up((size_t)num_requests * sizeof(SpecPlan), 256);
  *sub_off = *draw_off + align_up((size_t)num_requests * nvch * sizeof(double2), 256);
}

size_t draft_sub_offset(int num_requests, int vocab) {
  const size_t nvch = (size_t)((vocab + kVocabChunk - 1) / kVocabChunk);
  return align_up((size_t)num_requests * nvch * sizeof(MS), 256);
}

int launch_commit(const int32_t* req_ids, int batch, int num_requests, int k, const int32_t* n_out,
                  int32_t* seq_lens, int64_t* stats, cudaStream_t stream) {
  launch_pdl(commit_kernel, (batch + 255) / 256, 256, 0, stream, req_ids, batch, num_requests, k, n_out,
             seq_lens, reinterpret_cast<long long*>(stats));
  return cuda_status(cudaGetLastError(), __func__);
}

int launch_philox(uint64_t seed, int stream_id, const int32_t* request, const int32_t* position,
                  int64_t n, uint32_t* words, float* u, cudaStream_t stream) {
  launch_pdl(philox_kernel, (unsigned)((n + 255) / 256), 256, 0, stream, seed, stream_id, request, position,
                                                                 n, words, u);
  return cuda_status(cudaGetLastError(), __func__);
}

}  // namespace s3r
