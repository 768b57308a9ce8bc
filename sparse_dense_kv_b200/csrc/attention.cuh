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

template <int D, int NTW>
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
  // addresses). `visible(tile_row, nt, j)` says whether the lane's row j (0/1) of n-tile nt
  // sees the position in tile row `tile_row`; `capture(tile_row, nt, j, logit)` receives the
  // natural-log logit of every pair (visible or not).
  template <class Visible, class Capture>
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
      ldsm_x4(kb + swz(krow, 2 * ks + (mi >> 1)), a);
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) mma_bf16(s[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
    }
    const int p0 = row0 + (lane >> 2), p1 = p0 + 8;
    const float scale2 = scale * kLog2e;
    uint32_t b[NTW][2];
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt) {
      float x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int pr = (i < 2) ? p0 : p1;
        const int j = i & 1;
        capture(pr, nt, j, s[nt][i] * scale);
        x[i] = visible(pr, nt, j) ? s[nt][i] * scale2 : -INFINITY;
      }
      float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
      }
      const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
      const float al0 = (mn0 == -INFINITY) ? 1.f : ex2(m[nt][0] - mn0);
      const float al1 = (mn1 == -INFINITY) ? 1.f : ex2(m[nt][1] - mn1);
      m[nt][0] = mn0;
      m[nt][1] = mn1;
      const float e0 = (mn0 == -INFINITY) ? 0.f : ex2(x[0] - mn0);
      const float e1 = (mn1 == -INFINITY) ? 0.f : ex2(x[1] - mn1);
      const float e2 = (mn0 == -INFINITY) ? 0.f : ex2(x[2] - mn0);
      const float e3 = (mn1 == -INFINITY) ? 0.f : ex2(x[3] - mn1);
      l[nt][0] = l[nt][0] * al0 + e0 + e2;
      l[nt][1] = l[nt][1] * al1 + e1 + e3;
#pragma unroll
      for (int dm = 0; dm < D / 16; ++dm) {
        o[dm][nt][0] *= al0;
        o[dm][nt][1] *= al1;
        o[dm][nt][2] *= al0;
        o[dm][nt][3] *= al1;
      }
      b[nt][0] = movm_t(pack_bf16(e0, e1));
      b[nt][1] = movm_t(pack_bf16(e2, e3));
    }
    const int vrow = row0 + rr + 8 * (mi >> 1);
#pragma unroll
    for (int dm = 0; dm < D / 16; ++dm) {
      uint32_t a[4];
      ldsm_x4_t(vb + swz(vrow, 2 * dm + (mi & 1)), a);
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
template <int D, int RW>
__device__ __forceinline__ void merge_slices_to_record(const float* redO, const float* redM,
                                                       const float* redL, int ngroups,
                                                       float* rec, int Rp) {
  constexpr int DS = D + 4;
  const int rows = ngroups * RW;
  for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x) {
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

// Combine `nch` chunk records of `R` rows into normalised outputs: for row < R and d < D,
// out = sum_c O_c exp2(m_c - M) / sum_c l_c exp2(m_c - M); lse (natural) per row.
template <int D, class OutPtr, class LsePtr>
__device__ __forceinline__ void combine_records(const float* recs, size_t rec_floats, int nch,
                                                int R, int Rp, OutPtr out_row, LsePtr lse_row) {
  for (int idx = threadIdx.x; idx < R * D; idx += blockDim.x) {
    const int row = idx / D, d = idx - row * D;
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(recs + c * rec_floats + row));
    float acc = 0.f, lsum = 0.f;
    for (int c = 0; c < nch; ++c) {
      const float* rc = recs + c * rec_floats;
      const float mc = __ldcg(rc + row);
      const float f = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
      acc += f * __ldcg(rc + 2 * Rp + (size_t)row * D + d);
      lsum += f * __ldcg(rc + Rp + row);
    }
    out_row(row)[d] = __float2bfloat16_rn(acc / lsum);
    if (d == 0) {
      float* lp = lse_row(row);
      if (lp) *lp = (M + log2f(lsum)) * kLn2;
    }
  }
}

}  // namespace s3r
