// Shared warp-level attention machinery of the verify and draft kernels.
//
// Both kernels stream KV tiles of 64 positions into shared memory ([d/64][64][128 B],
// 128-byte swizzle) and compute the transposed products on the tensor cores:
//   S^T (16 positions x 8 rows) = K (16 x d) . Q^T (d x 8)      mma.m16n8k16, K from ldmatrix
//   O^T (d x 8 rows)           += V^T (d x 16) . P^T (16 x 8)    V^T from ldmatrix.trans
// P^T comes straight from the S^T accumulators: two floats -> bf16x2, then movmatrix.trans
// turns the accumulator layout into the B-operand layout, so P never touches shared memory.
// Each warp owns 16 positions of a tile and NTW n-tiles (8 rows each) and keeps its own
// online-softmax state in log2 units; warps are merged at the end of a chunk, chunks by the
// last CTA of a (request, KV head).
#pragma once

#include "common.cuh"

namespace s3r {

// Shared-memory layouts of a KV stage: byte offset of 16-byte chunk c of tile row `row`.
// Swz128: [d/64][64 rows][128 B] with the 128-byte swizzle (what a swizzled TMA box writes).
struct Swz128Layout {
  __device__ __forceinline__ static uint32_t off(int row, int c) { return swz(row, c); }
};
template <int D, int NTW, class Layout = Swz128Layout>
struct WarpAttn {
  uint32_t qf[NTW][D / 16][2];  // Q^T B-fragments
  float o[D / 16][NTW][4];      // O^T accumulators: (d = dm*16 + lane/4 (+8), row pair)
  float m[NTW][2];              // running max (log2 units) of the lane's two rows per n-tile
  float l[NTW][2];              // this lane's share of the row sums

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int dm = 0; dm < D / 16; ++dm)
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[dm][nt][i] = 0.f;
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
    }
  }

  // Q rows for n-tile nt: `qrow(row)` returns a pointer to the d bf16 values of tile row
  // `row` (0..7) or nullptr for a padding row.
  template <class RowPtr>
  __device__ __forceinline__ void load_q(int nt, int lane, RowPtr qrow) {
    const __nv_bfloat16* src = qrow(lane >> 2);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int d0 = ks * 16 + 2 * (lane & 3);
      qf[nt][ks][0] = src ? *reinterpret_cast<const uint32_t*>(src + d0) : 0u;
      qf[nt][ks][1] = src ? *reinterpret_cast<const uint32_t*>(src + d0 + 8) : 0u;
    }
  }

  // One 16-position m-tile starting at tile row `row0` of the stage at kb / vb (shared
  // addresses). With MASKED, `visible(tile_row, nt, j)` says whether the lane's row j (0/1)
  // of n-tile nt sees the position in tile row `tile_row` (without it every pair is
  // visible). `capture(tile_row, nt, logit_j0, logit_j1)` receives the natural-log logits
  // of the lane's two rows at each of its two positions.
  //
  // The running max is lazy: P = 2^(x - m) is formed against a reference max m that is
  // raised only when a tile exceeds it by more than 8 (log2 units), so P <= 256 stays exact
  // enough in bf16 and the O / l rescale is skipped for almost every tile.
  template <bool MASKED, class Visible, class Capture>
  __device__ __forceinline__ void step(uint32_t kb, uint32_t vb, int row0, int lane,
                                       float scale, Visible visible, Capture capture) {
    const int mi = lane >> 3, rr = lane & 7;
    float s[NTW][4];
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) s[nt][i] = 0.f;
    const int krow = row0 + rr + 8 * (mi & 1);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4(kb + Layout::off(krow, 2 * ks + (mi >> 1)), a);
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) mma_bf16(s[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
    }
    const int p0 = row0 + (lane >> 2), p1 = p0 + 8;
    const float scale2 = scale * kLog2e;
    uint32_t b[NTW][2];
    float al[NTW][2];
    bool any_rescale = false;
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt) {
      capture(p0, nt, s[nt][0] * scale, s[nt][1] * scale);
      capture(p1, nt, s[nt][2] * scale, s[nt][3] * scale);
      float x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[i] = s[nt][i] * scale2;
        if (MASKED && !visible((i < 2) ? p0 : p1, nt, i & 1)) x[i] = -INFINITY;
      }
      float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
      }
      al[nt][0] = al[nt][1] = 1.f;
      if (mx0 > m[nt][0] + 8.f) {
        al[nt][0] = ex2(m[nt][0] - mx0);   // 0 when m was -inf
        m[nt][0] = mx0;
        any_rescale = true;
      }
      if (mx1 > m[nt][1] + 8.f) {
        al[nt][1] = ex2(m[nt][1] - mx1);
        m[nt][1] = mx1;
        any_rescale = true;
      }
      const float r0 = m[nt][0], r1 = m[nt][1];
      const float e0 = (r0 == -INFINITY) ? 0.f : ex2(x[0] - r0);
      const float e1 = (r1 == -INFINITY) ? 0.f : ex2(x[1] - r1);
      const float e2 = (r0 == -INFINITY) ? 0.f : ex2(x[2] - r0);
      const float e3 = (r1 == -INFINITY) ? 0.f : ex2(x[3] - r1);
      l[nt][0] = l[nt][0] * al[nt][0] + e0 + e2;
      l[nt][1] = l[nt][1] * al[nt][1] + e1 + e3;
      b[nt][0] = movm_t(pack_bf16(e0, e1));
      b[nt][1] = movm_t(pack_bf16(e2, e3));
    }
    if (__any_sync(kFull, any_rescale)) {
#pragma unroll
      for (int dm = 0; dm < D / 16; ++dm)
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
          o[dm][nt][0] *= al[nt][0];
          o[dm][nt][1] *= al[nt][1];
          o[dm][nt][2] *= al[nt][0];
          o[dm][nt][3] *= al[nt][1];
        }
    }
    const int vrow = row0 + rr + 8 * (mi >> 1);
#pragma unroll
    for (int dm = 0; dm < D / 16; ++dm) {
      uint32_t a[4];
      ldsm_x4_t(vb + Layout::off(vrow, 2 * dm + (mi & 1)), a);
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) mma_bf16(o[dm][nt], a, b[nt][0], b[nt][1]);
    }
  }

  // Sum the lanes' row-sum shares (lanes with equal lane%4 hold the same rows).
  __device__ __forceinline__ void finish_sums() {
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float v = l[nt][j];
        v += __shfl_xor_sync(kFull, v, 4);
        v += __shfl_xor_sync(kFull, v, 8);
        v += __shfl_xor_sync(kFull, v, 16);
        l[nt][j] = v;
      }
  }

  // Write this warp's (m, l, O) for its 8*NTW rows into shared scratch slot `slot`:
  // redO [slots][8*NTW][D+4], redM / redL [slots][8*NTW].
  __device__ __forceinline__ void store_shared(float* redO, float* redM, float* redL, int slot,
                                               int lane) {
    constexpr int RW = 8 * NTW, DS = D + 4;
    float* ob = redO + (size_t)slot * RW * DS;
#pragma unroll
    for (int dm = 0; dm < D / 16; ++dm)
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int d = dm * 16 + (lane >> 2) + 8 * (i >> 1);
          const int row = nt * 8 + 2 * (lane & 3) + (i & 1);
          ob[row * DS + d] = o[dm][nt][i];
        }
    if (lane < 4) {
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int row = nt * 8 + 2 * lane + j;
          redM[slot * RW + row] = m[nt][j];
          redL[slot * RW + row] = l[nt][j];
        }
    }
  }
};

// Merge the 4 position-slice warps of each row group in shared scratch into one chunk
// record in global memory: rec = [m: Rp][l: Rp][O: Rp][D] (floats, m in log2 units).
// Warp w = group*4 + slice; group g covers rows g*RW .. g*RW+RW-1.
// Threads tid = 0..nthreads-1 share the work.
template <int D, int RW>
__device__ __forceinline__ void merge_slices_to_record(const float* redO, const float* redM,
                                                       const float* redL, int ngroups,
                                                       float* rec, int Rp, int tid, int nthreads) {
  constexpr int DS = D + 4;
  const int rows = ngroups * RW;
  for (int idx = tid; idx < rows * D; idx += nthreads) {
    const int grow = idx / D, d = idx - grow * D;
    const int g = grow / RW, rl = grow - g * RW;
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < 4; ++s) M = fmaxf(M, redM[(g * 4 + s) * RW + rl]);
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int slot = g * 4 + s;
      const float ms = redM[slot * RW + rl];
      const float f = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
      acc += f * redO[((size_t)slot * RW + rl) * DS + d];
      lsum += f * redL[slot * RW + rl];
    }
    rec[2 * Rp + (size_t)grow * D + d] = acc;
    if (d == 0) {
      rec[grow] = M;
      rec[Rp + grow] = lsum;
    }
  }
}

template <int D, int RW>
__device__ __forceinline__ void merge_slices_to_record(const float* redO, const float* redM,
                                                       const float* redL, int ngroups,
                                                       float* rec, int Rp) {
  merge_slices_to_record<D, RW>(redO, redM, redL, ngroups, rec, Rp, threadIdx.x, blockDim.x);
}

// Combine `nch` chunk records of `R` rows into normalised outputs: for row < R and d < D,
// out = sum_c O_c exp2(m_c - M) / sum_c l_c exp2(m_c - M); lse (natural) per row.
// Per-(chunk, row) weights go to shared memory (`wts`, capacity `wcap` floats) when they fit;
// otherwise each weight is recomputed from the record. Every thread then sums 4 consecutive
// d of one row over the chunks with 16-byte loads and writes them as bf16.
template <int D, class OutPtr, class LsePtr, class Sync>
__device__ __forceinline__ void combine_records_sync(const float* recs, size_t rec_floats,
                                                     int nch, int R, int Rp, float* wts, int wcap,
                                                     OutPtr out_row, LsePtr lse_row, int tid,
                                                     int nthreads, Sync sync) {
  float* Ms = wts;            // [R] row max
  float* iLs = wts + R;       // [R] 1 / row sum
  float* W = wts + 2 * R;     // [nch][R] weights, if they fit
  const bool table = (size_t)(2 + nch) * R <= (size_t)wcap;
  for (int row = tid; row < R; row += nthreads) {
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(recs + c * rec_floats + row));
    float lsum = 0.f;
    for (int c = 0; c < nch; ++c) {
      const float mc = __ldcg(recs + c * rec_floats + row);
      lsum += (mc == -INFINITY) ? 0.f : exp2f(mc - M) * __ldcg(recs + c * rec_floats + Rp + row);
    }
    Ms[row] = M;
    iLs[row] = 1.f / lsum;
    if (table)
      for (int c = 0; c < nch; ++c) {
        const float mc = __ldcg(recs + c * rec_floats + row);
        W[c * R + row] = (mc == -INFINITY) ? 0.f : exp2f(mc - M) / lsum;
      }
    float* lp = lse_row(row);
    if (lp) *lp = (M + log2f(lsum)) * kLn2;
  }
  sync();
  const int nvec = R * (D / 4);
  for (int v = tid; v < nvec; v += nthreads) {
    const int row = v / (D / 4), d4 = v - row * (D / 4);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int c = 0; c < nch; ++c) {
      float w;
      if (table) {
        w = W[c * R + row];
      } else {
        const float mc = __ldcg(recs + c * rec_floats + row);
        w = (mc == -INFINITY) ? 0.f : exp2f(mc - Ms[row]) * iLs[row];
      }
      const float4 x = __ldcg(reinterpret_cast<const float4*>(
          recs + c * rec_floats + 2 * Rp + (size_t)row * D) + d4);
      a.x += w * x.x;
      a.y += w * x.y;
      a.z += w * x.z;
      a.w += w * x.w;
    }
    __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(out_row(row) + d4 * 4);
    o[0] = __floats2bfloat162_rn(a.x, a.y);
    o[1] = __floats2bfloat162_rn(a.z, a.w);
  }
}

// combine_records_sync for a whole CTA (block-wide barriers).
template <int D, class OutPtr, class LsePtr>
__device__ __forceinline__ void combine_records(const float* recs, size_t rec_floats, int nch,
                                                int R, int Rp, float* wts, int wcap,
                                                OutPtr out_row, LsePtr lse_row, int tid,
                                                int nthreads) {
  combine_records_sync<D>(recs, rec_floats, nch, R, Rp, wts, wcap, out_row, lse_row, tid,
                          nthreads, [] { __syncthreads(); });
}

}  // namespace s3r
