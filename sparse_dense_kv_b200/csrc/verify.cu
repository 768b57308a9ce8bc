// Dense verify attention with score capture.
//
// What it computes ([News] Interpretation: the proposed block is recomputed against the
// complete historical KV; [Explainer] walkthrough: the sparse set comes from the verifier's
// last attention pass): for request r with committed length L and KV head h, the G*(k+1)
// rows (t, g) at positions L+t attend positions 0..L+t of the paged cache; the output,
// the log-sum-exp and every committed logit are written.
//
// Layout of the work: grid (chunk, kv_head, request). A CTA streams one chunk of `chunk`
// positions in tiles of 64: committed pages arrive by 2-D TMA (one 16-row box per page and
// 64-column half, 128-byte swizzle) into a 3-stage mbarrier pipeline; the block's own K/V
// (positions >= L) are patched into the tile from the caller's k_new / v_new. Warp
// (group, slice) computes 16 rows x 16 positions per tile on the tensor cores. Chunk
// results go to the workspace; verify_combine_kernel merges them in chunk order
// (deterministic) and writes out / lse.
#include "attention.cuh"
#include "kernels.h"

namespace s3r {

constexpr int kVerifyStages = 3;

template <int D>
constexpr int verify_stage_bytes() { return 2 * kTile * D * 2; }

template <int D, int MAXT>
__global__ void __launch_bounds__(MAXT) verify_kernel(const __grid_constant__ CUtensorMap tmK,
                                                     const __grid_constant__ CUtensorMap tmV,
                                                     const VerifyParams p) {
  pdl_wait();
  constexpr int NTW = 2, RW = 16, STAGE = verify_stage_bytes<D>();
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kVerifyStages * STAGE);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = warp >> 2, slice = warp & 3;
  const int bl = blockIdx.z, kvh = blockIdx.y, c = blockIdx.x;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) {
    if (c == 0 && kvh == 0 && tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int L = p.seq_lens[r];
  const int T = p.T, G = p.G, Lc = L + T;
  if (L < 0 || Lc > p.cap) {
    if (c == 0 && tid == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    return;
  }
  const int start = c * p.chunk;
  if (start >= Lc) return;
  const int end = min(start + p.chunk, Lc);
  const int* ptab = p.page_table + (size_t)r * p.max_pages;
  const int64_t npages = p.num_pages;
  const int Hkv = p.Hkv;

  // The block's K/V enter the cache (nothing in this launch reads them back from the pool).
  if (c == 0) {
    for (int idx = tid; idx < T * (D / 8); idx += blockDim.x) {
      const int t = idx / (D / 8), ch = idx - t * (D / 8);
      const int pos = L + t;
      const int page = ptab[pos >> 4];
      if (page < 0 || page >= npages) {
        set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
        continue;
      }
      const size_t dst = (((size_t)page * Hkv + kvh) * kPage + (pos & 15)) * D + ch * 8;
      const size_t src = (((size_t)r * T + t) * Hkv + kvh) * D + ch * 8;
      *reinterpret_cast<uint4*>(p.k_pool + dst) = *reinterpret_cast<const uint4*>(p.k_new + src);
      *reinterpret_cast<uint4*>(p.v_pool + dst) = *reinterpret_cast<const uint4*>(p.v_new + src);
    }
  }

  WarpAttn<D, NTW> wa;
  wa.init();
#pragma unroll
  for (int nt = 0; nt < NTW; ++nt) {
    const int base_row = grp * RW + nt * 8;
    wa.load_q(nt, lane, [&](int rr) -> const __nv_bfloat16* {
      const int row = base_row + rr;
      if (row >= p.R) return nullptr;
      const int t = row / G, g = row - t * G;
      return p.q + (((size_t)r * T + t) * p.Hq + kvh * G + g) * D;
    });
  }

  if (tid == 0) {
    for (int s = 0; s < kVerifyStages; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
    fence_proxy_async();
  }
  __syncthreads();

  const int ntiles = (end - start + kTile - 1) / kTile;
  const uint32_t sbase = smem_u32(smem);

  auto page_ok = [&](int pg) -> bool {
    const int id = ptab[pg];
    return id >= 0 && id < npages;
  };
  auto issue = [&](int it) {
    const int s = it % kVerifyStages;
    const int t0 = start + it * kTile;
    const uint32_t kdst = sbase + s * STAGE, vdst = kdst + kTile * D * 2;
    const uint32_t bar = smem_u32(&bars[s]);
    int ids[4];
    int nload = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int pg = (t0 >> 4) + i;
      ids[i] = -1;
      if (pg * kPage < L) {
        const int id = ptab[pg];
        if (id >= 0 && id < npages) {
          ids[i] = id;
          ++nload;
        } else {
          set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
        }
      }
    }
    mbar_arrive_expect_tx(bar, (uint32_t)(nload * kPage * D * 2 * 2));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (ids[i] < 0) continue;
      const int y = (int)(((int64_t)ids[i] * Hkv + kvh) * kPage);
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        tma_load_2d(kdst + h * kTile * 128 + i * kPage * 128, &tmK, h * 64, y, bar);
        tma_load_2d(vdst + h * kTile * 128 + i * kPage * 128, &tmV, h * 64, y, bar);
      }
    }
  };

  if (tid == 0)
    for (int s = 0; s < kVerifyStages - 1 && s < ntiles; ++s) issue(s);

  float* scores = p.scores;
  const int R = p.R;
  const size_t score_base = ((size_t)r * Hkv + kvh) * (size_t)p.cap * R;
  bool timed_out = false;

  for (int it = 0; it < ntiles; ++it) {
    if (tid == 0 && it + kVerifyStages - 1 < ntiles) issue(it + kVerifyStages - 1);
    const int s = it % kVerifyStages;
    const int t0 = start + it * kTile;
    const uint32_t kb = sbase + s * STAGE, vb = kb + kTile * D * 2;
    if (!mbar_wait(smem_u32(&bars[s]), (it / kVerifyStages) & 1)) timed_out = true;

    // Patch rows the TMA did not bring: the block (from k_new / v_new), rows past the
    // context and rows of a page id outside the pool (zeros).
    bool fix = (t0 + kTile > L);
    if (!fix) {
#pragma unroll
      for (int i = 0; i < 4; ++i) fix |= !page_ok((t0 >> 4) + i);
    }
    if (fix) {
      uint8_t* kst = smem + s * STAGE;
      uint8_t* vst = kst + kTile * D * 2;
      for (int idx = tid; idx < 2 * kTile * (D / 8); idx += blockDim.x) {
        const int which = idx / (kTile * (D / 8));
        const int rem = idx - which * (kTile * (D / 8));
        const int row = rem / (D / 8), ch = rem - row * (D / 8);
        const int pos = t0 + row;
        if (pos < L && page_ok(pos >> 4)) continue;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (pos >= L && pos < Lc) {
          const size_t src = (((size_t)r * T + (pos - L)) * Hkv + kvh) * D + ch * 8;
          v = *reinterpret_cast<const uint4*>((which ? p.v_new : p.k_new) + src);
        }
        *reinterpret_cast<uint4*>((which ? vst : kst) + swz(row, ch)) = v;
      }
      fence_proxy_async();
      __syncthreads();
    }

    const int row0 = slice * 16;
    if (t0 + row0 < end) {
      auto vis = [&](int tr, int nt, int j) -> bool {
        const int pos = t0 + tr;
        const int row = grp * RW + nt * 8 + 2 * (lane & 3) + j;
        return pos < end && (pos < L || pos - L <= row / G);
      };
      auto cap_fn = [&](int tr, int nt, float lg0, float lg1) {
        const int pos = t0 + tr;
        const int row = grp * RW + nt * 8 + 2 * (lane & 3);
        if (scores && row < R && pos < L) {   // [row][position]
          float* dst = scores + score_base + (size_t)row * p.cap + pos;
          dst[0] = lg0;
          if (row + 1 < R) dst[p.cap] = lg1;
        }
      };
      if (t0 + kTile <= L && t0 + kTile <= end)
        wa.template step<false>(kb, vb, row0, lane, p.scale, vis, cap_fn);
      else
        wa.template step<true>(kb, vb, row0, lane, p.scale, vis, cap_fn);
    }
    if (__syncthreads_or(timed_out)) {
      if (tid == 0) set_error(p.err, S3R_ERR_TIMEOUT);
      // drain: give copies already issued a bounded chance to land before leaving
      for (int k2 = it + 1; k2 < min(ntiles, it + kVerifyStages); ++k2)
        mbar_wait(smem_u32(&bars[k2 % kVerifyStages]), (k2 / kVerifyStages) & 1);
      return;
    }
  }

  wa.finish_sums();
  // Shared scratch for the slice merge reuses the pipeline stages.
  const int nwarps = blockDim.x >> 5;
  float* redO = reinterpret_cast<float*>(smem);
  float* redM = redO + (size_t)nwarps * RW * (D + 4);
  float* redL = redM + nwarps * RW;
  wa.store_shared(redO, redM, redL, warp, lane);
  __syncthreads();
  const size_t rec_floats = (size_t)p.Rp * (D + 2);
  float* recs = p.part + ((size_t)r * Hkv + kvh) * p.nchunk_max * rec_floats;
  merge_slices_to_record<D, RW>(redO, redM, redL, nwarps / 4, recs + c * rec_floats, p.Rp);

}

// Merge the chunk records of every (request, KV head) of a verify launch into out / lse.
// Grid (group of kCombRows rows, KV head, request), so a launch has a few CTAs per SM and
// every merge runs at once: the group's chunk maxima / sums are loaded in one round (with
// the first batch of output slices, which do not depend on them), the weights of each row
// are formed in shared memory, then every thread accumulates two 16-byte output slices over
// the chunks in chunk order with kCombBatch chunks' loads in flight. kCombMinBlocks CTAs
// fit an SM, so the 32-request Qwen3-8B launch (1024 CTAs) is one wave.
constexpr int kCombRows = 8;
constexpr int kCombThreads = 128;
constexpr int kCombBatch = 4;   // chunks whose loads are issued together
constexpr int kCombMinBlocks = 7;

template <int D>
__global__ void __launch_bounds__(kCombThreads, kCombMinBlocks) verify_combine_kernel(const VerifyParams p) {
  pdl_wait();
  extern __shared__ float cw[];   // m, l, weights: [nch][kCombRows] each
  const int j0 = blockIdx.x * kCombRows, kvh = blockIdx.y, bl = blockIdx.z;
  const int r = p.req_ids ? p.req_ids[bl] : bl;
  if (r < 0 || r >= p.num_requests) return;     // bad ids are reported by the attention kernel
  const int L = p.seq_lens[r];
  const int T = p.T, G = p.G, R = p.R, Rp = p.Rp, Lc = L + T;
  if (L < 0 || Lc > p.cap || j0 >= R) return;   // bad lengths are reported by the attention kernel
  const int nr = min(kCombRows, R - j0);
  const int nch = (Lc + p.chunk - 1) / p.chunk;
  const size_t rec_floats = (size_t)Rp * (D + 2);
  const float* recs = p.part + ((size_t)r * p.Hkv + kvh) * p.nchunk_max * rec_floats;
  float* mm = cw;
  float* ll = cw + (size_t)nch * kCombRows;
  float* ww = ll + (size_t)nch * kCombRows;
  constexpr int kQ = D / 4;       // float4 slices per row
  const int nvec = nr * kQ;
  // this thread's first output slices (v0, v0 + blockDim.x) and their first batch of chunks
  const int v0f = threadIdx.x, v1f = v0f + blockDim.x;
  const float4* recO = reinterpret_cast<const float4*>(recs + 2 * Rp + (size_t)j0 * D);
  float4 xa[kCombBatch], xb[kCombBatch];
  const int nb0 = min(kCombBatch, nch);
  if (v0f < nvec) {
#pragma unroll
    for (int u = 0; u < kCombBatch; ++u) {
      if (u < nb0) {
        const size_t off = (size_t)u * rec_floats / 4;
        xa[u] = __ldcg(recO + v0f + off);
        xb[u] = __ldcg(recO + (v1f < nvec ? v1f : v0f) + off);
      }
    }
  }
  for (int i = threadIdx.x; i < nch * nr; i += blockDim.x) {
    const int c = i / nr, j = i - c * nr;
    mm[c * kCombRows + j] = __ldcg(recs + c * rec_floats + j0 + j);
    ll[c * kCombRows + j] = __ldcg(recs + c * rec_floats + Rp + j0 + j);
  }
  __syncthreads();
  if (threadIdx.x < nr) {
    const int j = threadIdx.x, row = j0 + j;
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, mm[c * kCombRows + j]);
    float lsum = 0.f;
    for (int c = 0; c < nch; ++c) {
      const float mc = mm[c * kCombRows + j];
      lsum += (mc == -INFINITY) ? 0.f : exp2f(mc - M) * ll[c * kCombRows + j];
    }
    const float inv = 1.f / lsum;
    for (int c = 0; c < nch; ++c) {
      const float mc = mm[c * kCombRows + j];
      ww[c * kCombRows + j] = (mc == -INFINITY) ? 0.f : exp2f(mc - M) * inv;
    }
    const int t = row / G, g = row - t * G;
    p.lse[((size_t)r * T + t) * p.Hq + kvh * G + g] = (M + log2f(lsum)) * kLn2;
  }
  __syncthreads();
  for (int v0 = threadIdx.x; v0 < nvec; v0 += 2 * blockDim.x) {
    const int v1 = v0 + blockDim.x;
    const bool has1 = v1 < nvec;
    const int ja = v0 / kQ, jb = has1 ? v1 / kQ : ja;
    const float4* pa = recO + v0;
    const float4* pb = recO + (has1 ? v1 : v0);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    for (int c0 = 0; c0 < nch; c0 += kCombBatch) {
      const int nb = min(kCombBatch, nch - c0);
      if (v0 != v0f || c0 > 0) {   // the first batch of the first slices was loaded above
#pragma unroll
        for (int u = 0; u < kCombBatch; ++u) {
          if (u < nb) {
            const size_t off = (size_t)(c0 + u) * rec_floats / 4;
            xa[u] = __ldcg(pa + off);
            xb[u] = __ldcg(pb + off);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kCombBatch; ++u) {
        if (u < nb) {
          const float wa = ww[(c0 + u) * kCombRows + ja], wb = ww[(c0 + u) * kCombRows + jb];
          a.x += wa * xa[u].x;
          a.y += wa * xa[u].y;
          a.z += wa * xa[u].z;
          a.w += wa * xa[u].w;
          b.x += wb * xb[u].x;
          b.y += wb * xb[u].y;
          b.z += wb * xb[u].z;
          b.w += wb * xb[u].w;
        }
      }
    }
    auto store = [&](int v, int j, const float4& acc) {
      const int row = j0 + j, d4 = v - j * kQ;
      const int t = row / G, g = row - t * G;
      __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(
          p.out + (((size_t)r * T + t) * p.Hq + kvh * G + g) * D + d4 * 4);
      o[0] = __floats2bfloat162_rn(acc.x, acc.y);
      o[1] = __floats2bfloat162_rn(acc.z, acc.w);
    };
    store(v0, ja, a);
    if (has1) store(v1, jb, b);
  }
}

bool verify_combine_fits(int nchunk_max, int /*R*/) {
  return (size_t)3 * nchunk_max * kCombRows * 4 <= 200 * 1024;
}

int launch_verify_combine(const VerifyParams& p, int D, int batch, cudaStream_t stream) {
  const size_t smem = (size_t)3 * p.nchunk_max * kCombRows * 4;
  if (!verify_combine_fits(p.nchunk_max, p.R)) return S3R_ERR_UNSUPPORTED;
  dim3 grid((p.R + kCombRows - 1) / kCombRows, p.Hkv, batch);
  auto kern = D == 128 ? verify_combine_kernel<128> : verify_combine_kernel<64>;
  // the limit is raised once per device to the largest merge that verify_combine_fits admits
  static std::atomic<uint64_t> attr_done[2];
  if (smem > 48 * 1024 &&
      cuda_status(ensure_smem_attr(kern, 200 * 1024, attr_done[D == 128 ? 0 : 1]), "cudaFuncSetAttribute") != S3R_OK)
    return S3R_ERR_CUDA;
  launch_pdl(kern, grid, kCombThreads, smem, stream, p);
  return cuda_status(cudaGetLastError(), __func__);
}

template <int D, int MAXT>
static int launch_verify_t(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyParams& p,
                           int batch, cudaStream_t stream) {
  const int ngroups = (p.R + 15) / 16;
  const int threads = 128 * ngroups;
  const size_t smem = 1024 + kVerifyStages * verify_stage_bytes<D>() + 64;
  const size_t red = (size_t)(threads / 32) * 16 * (D + 4 + 2) * 4;
  const size_t need = smem > red + 1024 + 64 ? smem : red + 1024 + 64;
  // raised once per device to what the largest row count (S3R_MAX_ROWS: 4 row groups) needs
  const size_t red_max = (size_t)(128 * ((S3R_MAX_ROWS + 15) / 16) / 32) * 16 * (D + 4 + 2) * 4;
  const size_t need_max = smem > red_max + 1024 + 64 ? smem : red_max + 1024 + 64;
  static std::atomic<uint64_t> attr_done{0};
  if (cuda_status(ensure_smem_attr(verify_kernel<D, MAXT>, (int)need_max, attr_done), "cudaFuncSetAttribute") !=
      S3R_OK)
    return S3R_ERR_CUDA;
  dim3 grid(p.nchunk_max, p.Hkv, batch);
  launch_pdl(verify_kernel<D, MAXT>, grid, threads, need, stream, tk, tv, p);
  return cuda_status(cudaGetLastError(), __func__);
}

template <int D>
static int launch_verify_d(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyParams& p,
                           int batch, cudaStream_t stream) {
  if (p.R <= 32) return launch_verify_t<D, 256>(tk, tv, p, batch, stream);
  return launch_verify_t<D, 512>(tk, tv, p, batch, stream);
}

int launch_verify(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyParams& p, int D,
                  int batch, cudaStream_t stream) {
  if (D == 128) return launch_verify_d<128>(tk, tv, p, batch, stream);
  if (D == 64) return launch_verify_d<64>(tk, tv, p, batch, stream);
  return S3R_ERR_UNSUPPORTED;
}

size_t verify_partial_bytes(int num_requests, int Hkv, int cap, int R, int D, int chunk) {
  const int Rp = ((R + 15) / 16) * 16;
  const size_t nchunk = (size_t)((cap + chunk - 1) / chunk);
  return align_up((size_t)num_requests * Hkv * nchunk * Rp * (D + 2) * 4, 256);
}

}  // namespace s3r
