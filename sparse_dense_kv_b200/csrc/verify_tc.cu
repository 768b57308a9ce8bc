// Dense verify attention with score capture on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory), head_dim 128, up to 32 rows per KV head.
//
// What it computes is what verify.cu computes ([News] Interpretation: the proposed block is
// recomputed against the complete historical KV; [Explainer] walkthrough: the sparse set
// comes from the verifier's last attention pass): rows (t, g) at positions L+t attend
// positions 0..L+t; out, lse and every committed logit are written.
//
// Organisation (one persistent CTA per SM, 6 warps):
//   warp 0     producer: per work item (request, KV head, chunk of up to 8 tiles of 128
//              positions) it copies the item's Q rows into shared memory, then streams the
//              chunk's K tiles and then its V tiles through a 4-stage ring with 4-D TMA over
//              (d, slot, head, page): a tile of 8 consecutive page ids is 2 boxes (one per
//              64-column half, 128-byte swizzle), otherwise one box per page and half. The
//              tile holding the block (positions >= L) is patched after its TMA lands.
//   warp 1     MMA issuer: S^T tile t (128 positions x N rows, fp32) = K_t . Q^T into tensor
//              memory columns [t*N, t*N+N) for every tile of the chunk, then, once the
//              softmax warps have written P^T, O^T (128 d x N) = sum_t V_t^T . P_t^T into the
//              columns after them. K and Q are K-major operands (128-byte swizzle); V^T is
//              MN-major (the V tile as it arrives, 128-byte swizzle) and so is P^T (one row of
//              N values per position, 32- or 64-byte swizzle).
//   warps 2-5  softmax / epilogue (one thread per tensor-memory lane = position or d):
//              pass 1 reads every S tile, writes the committed logits and takes the chunk
//              maximum per row; pass 2 re-reads them and writes P = 2^(s - max) as bf16 P^T
//              tiles; then the chunk record (max, sum, O) goes to the workspace, and a small
//              second kernel merges the chunks of every (request, KV head).
// The softmax is exact per chunk (two passes over logits resident in tensor memory), so no
// running rescale exists; chunks merge by their (max, sum) as in the CUDA-core kernel.
#include "attention.cuh"
#include "kernels.h"

namespace s3r {
namespace tc {

constexpr int kPos = 128;                   // positions per tile (MMA M)
constexpr int kD = 128;                     // head_dim of this path
constexpr int kStages = 4;
constexpr int kThreads = 320;          // producer, MMA, 8 softmax warps
constexpr int kTileBytes = kPos * kD * 2;   // 32 KB: [2 halves][128 rows][128 B]
constexpr int kMaxBatch = 1024;             // requests per launch on this path

// --------------------------------------------------------------- tcgen05 wrappers -------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
// This warp's 32 lanes x 16 consecutive columns (one fp32 per column per thread).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N]) {
#pragma unroll
  for (int c = 0; c < N; c += 16) {
    float w[16];
    tmem_ld16(taddr + c, w);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[c + i] = w[i];
  }
}

// Shared-memory matrix descriptor: start, leading / stride byte offsets, sm100 version 1,
// swizzle layout (2 = 128 B, 4 = 64 B, 6 = 32 B).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                          uint32_t layout) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) |
         ((uint64_t)layout << 61);
}
// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, M x N, operand majors.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int NP>
struct Cfg {
  static constexpr int kTiles = NP == 32 ? 7 : 8;            // tiles per chunk
  static constexpr int kChunk = kTiles * kPos;
  static constexpr int kQBytes = 2 * NP * 128;               // [2 halves][NP rows][128 B]
  static constexpr int kPTile = kPos * NP * 2;               // P^T tile: [128 pos][NP rows] bf16
  static constexpr int kPBytes = kTiles * kPTile;
  static constexpr uint32_t kPSwz = NP == 16 ? 6u : 4u;      // 32- / 64-byte swizzle
  static constexpr int kTmemCols = 512;
  static constexpr int kSCols = kTiles * NP;                 // one S buffer
  static constexpr int kOCol = 2 * kSCols;                   // two O buffers after two S buffers
  static_assert(kOCol + 2 * NP <= kTmemCols, "tensor memory budget");
  static constexpr int kRingOff = 0;
  static constexpr int kQOff = kStages * kTileBytes;
  static constexpr int kPOff = kQOff + kQBytes;
  static constexpr int kRedOff = kPOff + kPBytes;            // redM, redL [8 warps][NP]; cm, cl [2][NP]
  static constexpr int kRedBytes = (2 * 8 * NP + 4 * NP) * 4;
  static constexpr int kPrefOff = kRedOff + kRedBytes;       // request prefix [kMaxBatch+1]
  static constexpr int kLenOff = kPrefOff + (kMaxBatch + 1) * 4;   // L per request [kMaxBatch]
  static constexpr int kRidOff = kLenOff + kMaxBatch * 4;          // request id [kMaxBatch]
  static constexpr int kIdsOff = kRidOff + kMaxBatch * 4;          // page ids [2 items][64]
  static constexpr int kBarOff = (kIdsOff + 2 * 64 * 4 + 63) / 64 * 64;
  static constexpr int kSmem = kBarOff + 256 + 1024;         // + barriers + alignment slack
};

struct Bars {
  uint64_t full[kStages], empty[kStages], tma[kStages];
  // one barrier pair per tensor-memory buffer (chunk parity), so that no barrier ever runs
  // two phases ahead of a waiter
  uint64_t q_full, q_empty, p_full, fin;
  uint64_t s_full[2], s_empty[2], o_full[2], o_empty[2];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Warp-uniform bounded wait on an mbarrier phase (every lane observes the phase itself).
// Gives up when another role raised the abort flag, or after kWaitLimit polls (then raises
// it, with S3R_ERR_TIMEOUT in the error word).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int* err) {
  for (int i = 0; i < kWaitLimit; ++i) {
    const bool done = mbar_try_wait(bar, parity);
    if (__all_sync(kFull, done)) return true;
    if ((i & 255) == 255 && __any_sync(kFull, *abort_flag != 0)) return false;
  }
  if ((threadIdx.x & 31) == 0) {
    *abort_flag = 1;
    set_error(err, S3R_ERR_TIMEOUT);
  }
  __syncwarp();
  return false;
}
__device__ __forceinline__ bool aborted(volatile int* abort_flag) {
  return __any_sync(kFull, *abort_flag != 0);
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void named_sync_softmax() {
  asm volatile("bar.sync 1, 256;\n" ::: "memory");
}

// Work item i of the launch -> (launch-local request, KV head, chunk), from the prefix of
// per-request item counts (items of request b = Hkv * chunks_b).
__device__ __forceinline__ void item_of(int i, const int* pref, int batch, int Hkv,
                                        int& bl, int& kvh, int& c) {
  int lo = 0, hi = batch;   // largest bl with pref[bl] <= i
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pref[mid] <= i) lo = mid;
    else hi = mid;
  }
  bl = lo;
  const int rem = i - pref[lo];
  const int nch = (pref[lo + 1] - pref[lo]) / Hkv;
  kvh = rem / nch;
  c = rem - kvh * nch;
}

struct Item {
  int r, kvh, c, L, Lc, start, end, ntile;
};

template <int NP>
__device__ __forceinline__ Item make_item(int it, const int* pref, const int* lens_s,
                                          const int* rid_s, int batch, const VerifyParams& p) {
  Item x;
  int bl;
  item_of(it, pref, batch, p.Hkv, bl, x.kvh, x.c);
  x.r = rid_s[bl];
  x.L = lens_s[bl];
  x.Lc = x.L + p.T;
  x.start = x.c * Cfg<NP>::kChunk;
  x.end = min(x.start + Cfg<NP>::kChunk, x.Lc);
  x.ntile = (x.end - x.start + kPos - 1) / kPos;
  return x;
}

template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
    verify_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmK8, const __grid_constant__ CUtensorMap tmV8,
                     const VerifyParams p, int batch) {
  using C = Cfg<NP>;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                             ~uintptr_t(1023));
  int* pref = reinterpret_cast<int*>(smem + C::kPrefOff);
  int* lens_s = reinterpret_cast<int*>(smem + C::kLenOff);
  int* rid_s = reinterpret_cast<int*>(smem + C::kRidOff);
  int* ids_s = reinterpret_cast<int*>(smem + C::kIdsOff);
  float* redM = reinterpret_cast<float*>(smem + C::kRedOff);   // [8][NP]
  float* redL = redM + 8 * NP;                                  // [8][NP]
  float* cm = redL + 8 * NP;                                    // [2][NP] chunk max (log2)
  float* cl = cm + 2 * NP;                                      // [2][NP] chunk sum
  Bars* B = reinterpret_cast<Bars*>(smem + C::kBarOff);
  volatile int* abort_flag = &B->abort_flag;
  __shared__ int trow[NP];   // block row t of query row j (j / G)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = p.T, G = p.G, R = p.R, Hkv = p.Hkv, Hq = p.Hq;
  const int chunk = C::kChunk;
  const uint32_t sbase = smem_u32(smem);

  // ---- set-up: request prefix (items), barriers, tensor memory
  for (int b = tid; b < batch; b += blockDim.x) {
    const int r = p.req_ids ? p.req_ids[b] : b;
    const int L = p.seq_lens[r];
    const int Lc = L + T;
    rid_s[b] = r;
    lens_s[b] = L;
    int items = 0;
    if (L >= 0 && Lc <= p.cap) items = Hkv * ((Lc + chunk - 1) / chunk);
    else if (blockIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    pref[b + 1] = items;
  }
  __syncthreads();
  if (warp == 0) {
    // inclusive scan of pref[1..batch]: lane l owns a contiguous segment
    const int per = (batch + 31) / 32;
    const int b0 = lane * per, b1 = min(batch, b0 + per);
    int local = 0;
    for (int b = b0; b < b1; ++b) local += pref[b + 1];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int b = b0; b < b1; ++b) {
      run += pref[b + 1];
      pref[b + 1] = run;
    }
    if (lane == 0) pref[0] = 0;
  }
  if (tid < NP) trow[tid] = tid / G;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&B->full[s]), 1);
      mbar_init(smem_u32(&B->empty[s]), 1);
      mbar_init(smem_u32(&B->tma[s]), 1);
    }
    mbar_init(smem_u32(&B->q_full), 1);
    mbar_init(smem_u32(&B->q_empty), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&B->s_full[b]), 1);
      mbar_init(smem_u32(&B->s_empty[b]), 8);
      mbar_init(smem_u32(&B->o_full[b]), 1);
      mbar_init(smem_u32(&B->o_empty[b]), 8);
    }
    mbar_init(smem_u32(&B->p_full), 8);
    mbar_init(smem_u32(&B->fin), 1);
    B->abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&B->tmem_base), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;
  const int nitems = pref[batch];
  const int my_items = nitems > (int)blockIdx.x ? (nitems - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const uint32_t qbuf = sbase + C::kQOff, pbuf = sbase + C::kPOff;

  if (warp == 0) {
    // ===================================================================== producer ====
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmK)) : "memory");
      asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmV)) : "memory");
      asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmK8)) : "memory");
      asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmV8)) : "memory");
    }
    // ring order: K(0), then per item n: K(n+1), V(n) -- the MMA warp consumes in this order
    int g = 0;
    uint32_t tma_phase = 0;   // bit s: phase of tma[s]
    bool stop = false;
    auto load_tiles = [&](const Item& x, bool is_v, const int* ids_item) {
      const CUtensorMap* map = is_v ? &tmV : &tmK;
      const CUtensorMap* map8 = is_v ? &tmV8 : &tmK8;
      const __nv_bfloat16* blk = is_v ? p.v_new : p.k_new;
      for (int t = 0; t < x.ntile && !stop; ++t, ++g) {
        const int s = g % kStages;
        if (g >= kStages &&
            !wait_bar(smem_u32(&B->empty[s]), ((g / kStages) - 1) & 1, abort_flag, p.err)) {
          stop = true;
          break;
        }
        const int t0 = x.start + t * kPos;
        const uint32_t dst = sbase + C::kRingOff + s * kTileBytes;
        uint32_t okmask = 0;
        int nload = 0;
        bool tail = (t0 + kPos > x.L);
        int ids[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) ids[i] = ids_item[t * 8 + i];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int pg = (t0 >> 4) + i;
          if (pg * kPage < x.L) {
            if (ids[i] >= 0 && ids[i] < p.num_pages) {
              okmask |= 1u << i;
              ++nload;
            } else {
              tail = true;
              if (lane == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
            }
          }
        }
        const uint32_t landing = smem_u32(tail ? &B->tma[s] : &B->full[s]);
        if (lane == 0) mbar_arrive_expect_tx(landing, (uint32_t)(nload * kPage * kD * 2));
        __syncwarp();
        bool run = okmask == 0xFFu && !tail;   // 8 consecutive page ids: 2 boxes of 8 pages
#pragma unroll
        for (int i = 1; i < 8; ++i) run = run && ids[i] == ids[0] + i;
        if (run) {
          if (lane < 2) tma_load_4d(dst + lane * kPos * 128, map8, lane * 64, 0, x.kvh, ids[0], landing);
        } else if (lane < 16) {
          // one page per lane pair (page lane/2, half lane%2)
          const int i = lane >> 1, h = lane & 1;
          if (okmask & (1u << i))
            tma_load_4d(dst + h * kPos * 128 + i * kPage * 128, map, h * 64, 0, x.kvh, ids[i], landing);
        }
        if (tail) {
          // wait for the committed rows, then write block rows / zeros over the rest
          if (!wait_bar(smem_u32(&B->tma[s]), (tma_phase >> s) & 1, abort_flag, p.err)) {
            stop = true;
            break;
          }
          tma_phase ^= 1u << s;
          for (int idx = lane; idx < kPos * (kD / 8); idx += 32) {
            const int row = idx / (kD / 8), ch = idx - row * (kD / 8);
            const int pos = t0 + row;
            if (pos < x.L && (okmask & (1u << (row >> 4)))) continue;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (pos >= x.L && pos < x.Lc)
              v = *reinterpret_cast<const uint4*>(blk + (((size_t)x.r * T + (pos - x.L)) * Hkv + x.kvh) * kD + ch * 8);
            const uint32_t off = (ch >> 3) * (kPos * 128) + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
            *reinterpret_cast<uint4*>(smem + C::kRingOff + s * kTileBytes + off) = v;
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&B->full[s]));
        }
        __syncwarp();
      }
    };
    auto load_q_and_k = [&](int m) {
      const Item x = make_item<NP>(blockIdx.x + m * gridDim.x, pref, lens_s, rid_s, batch, p);
      const int* ptab = p.page_table + (size_t)x.r * p.max_pages;
      // page ids of the item's committed pages (-1 past L), read once for its K and V tiles
      int* ids_item = ids_s + (m & 1) * 64;
      {
        const int npg = x.ntile * 8;
        const int pg0 = x.start >> 4;
        const int a = lane < npg && (pg0 + lane) * kPage < x.L ? ptab[pg0 + lane] : -1;
        const int b = lane + 32 < npg && (pg0 + lane + 32) * kPage < x.L ? ptab[pg0 + lane + 32] : -1;
        ids_item[lane] = a;
        ids_item[lane + 32] = b;
      }
      if (x.c == 0) {   // the block's K/V enter the cache once per (request, head)
        for (int idx = lane; idx < T * (kD / 8); idx += 32) {
          const int t = idx / (kD / 8), ch = idx - t * (kD / 8);
          const int pos = x.L + t;
          const int page = ptab[pos >> 4];
          if (page < 0 || page >= p.num_pages) {
            set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
            continue;
          }
          const size_t dst = (((size_t)page * Hkv + x.kvh) * kPage + (pos & 15)) * kD + ch * 8;
          const size_t src = (((size_t)x.r * T + t) * Hkv + x.kvh) * kD + ch * 8;
          *reinterpret_cast<uint4*>(p.k_pool + dst) = *reinterpret_cast<const uint4*>(p.k_new + src);
          *reinterpret_cast<uint4*>(p.v_pool + dst) = *reinterpret_cast<const uint4*>(p.v_new + src);
        }
      }
      // Q rows -> qbuf (K-major, 128-byte swizzle, zero padding rows), once QK(m-1) is done
      constexpr int kPer = NP * (kD / 8) / 32;
      uint4 qv[kPer];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int idx = lane + 32 * i;
        const int row = idx / (kD / 8), ch = idx - row * (kD / 8);
        qv[i] = make_uint4(0, 0, 0, 0);
        if (row < R) {
          const int t = row / G, gg = row - t * G;
          qv[i] = __ldg(reinterpret_cast<const uint4*>(
              p.q + (((size_t)x.r * T + t) * Hq + x.kvh * G + gg) * kD + ch * 8));
        }
      }
      if (m > 0 && !wait_bar(smem_u32(&B->q_empty), (m - 1) & 1, abort_flag, p.err)) {
        stop = true;
        return;
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int idx = lane + 32 * i;
        const int row = idx / (kD / 8), ch = idx - row * (kD / 8);
        const uint32_t off = (ch >> 3) * (NP * 128) + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(smem + C::kQOff + off) = qv[i];
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&B->q_full));
      load_tiles(x, false, ids_item);
    };
    if (my_items > 0) load_q_and_k(0);
    for (int n = 0; n < my_items && !stop && !aborted(abort_flag); ++n) {
      if (n + 1 < my_items) load_q_and_k(n + 1);
      if (stop) break;
      load_tiles(make_item<NP>(blockIdx.x + n * gridDim.x, pref, lens_s, rid_s, batch, p), true,
                 ids_s + (n & 1) * 64);
    }
  } else if (warp == 1) {
    // ====================================================================== MMA warp ===
    constexpr uint32_t kIdQK = idesc_bf16(kPos, NP, false, false);
    constexpr uint32_t kIdPV = idesc_bf16(kD, NP, true, true);
    int g = 0;
    bool ok = true;
    auto qk = [&](int m) {
      const Item x = make_item<NP>(blockIdx.x + m * gridDim.x, pref, lens_s, rid_s, batch, p);
      ok = wait_bar(smem_u32(&B->q_full), m & 1, abort_flag, p.err);
      if (ok && m >= 2) ok = wait_bar(smem_u32(&B->s_empty[m & 1]), ((m - 2) >> 1) & 1, abort_flag, p.err);
      if (!ok) return;
      tc_fence_after();
      const uint32_t sd = tmem + (m & 1) * C::kSCols;
      for (int t = 0; t < x.ntile; ++t, ++g) {
        const int s = g % kStages;
        ok = wait_bar(smem_u32(&B->full[s]), (g / kStages) & 1, abort_flag, p.err);
        if (!ok) return;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t kt = sbase + C::kRingOff + s * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t ad = sdesc(kt + (kk >> 2) * (kPos * 128) + (kk & 3) * 32, 16, 1024, 2);
            const uint64_t bd = sdesc(qbuf + (kk >> 2) * (NP * 128) + (kk & 3) * 32, 16, 1024, 2);
            tc_mma(sd + t * NP, ad, bd, kIdQK, kk > 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&B->empty[s]));
        }
        __syncwarp();
      }
      if (lane == 0) {
        tc_commit(smem_u32(&B->s_full[m & 1]));
        tc_commit(smem_u32(&B->q_empty));
      }
      __syncwarp();
    };
    auto pv = [&](int n) {
      const Item x = make_item<NP>(blockIdx.x + n * gridDim.x, pref, lens_s, rid_s, batch, p);
      ok = wait_bar(smem_u32(&B->p_full), n & 1, abort_flag, p.err);
      if (ok && n >= 2) ok = wait_bar(smem_u32(&B->o_empty[n & 1]), ((n - 2) >> 1) & 1, abort_flag, p.err);
      if (!ok) return;
      tc_fence_after();
      const uint32_t od = tmem + C::kOCol + (n & 1) * NP;
      for (int t = 0; t < x.ntile; ++t, ++g) {
        const int s = g % kStages;
        ok = wait_bar(smem_u32(&B->full[s]), (g / kStages) & 1, abort_flag, p.err);
        if (!ok) return;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t vt = sbase + C::kRingOff + s * kTileBytes;
          const uint32_t pt = pbuf + t * C::kPTile;
#pragma unroll
          for (int kk = 0; kk < kPos / 16; ++kk) {
            const uint64_t ad = sdesc(vt + kk * 2048, kPos * 128, 1024, 2);
            const uint64_t bd = sdesc(pt + kk * 16 * NP * 2, NP * 2 * 8, 8 * NP * 2, C::kPSwz);
            tc_mma(od, ad, bd, kIdPV, (t > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&B->empty[s]));
        }
        __syncwarp();
      }
      if (lane == 0) tc_commit(smem_u32(&B->o_full[n & 1]));
      __syncwarp();
    };
    if (my_items > 0) qk(0);
    for (int n = 0; n < my_items && ok && !aborted(abort_flag); ++n) {
      if (n + 1 < my_items) qk(n + 1);
      if (!ok) break;
      pv(n);
    }
    // make sure nothing issued is still running before the tensor memory goes away
    if (lane == 0) tc_commit(smem_u32(&B->fin));
    __syncwarp();
    wait_bar(smem_u32(&B->fin), 0, abort_flag, p.err);
  } else {
    // ================================================================ softmax warps ===
    const int sw8 = warp - 2;                // 0..7
    const int sg = sw8 >> 2;                 // warpgroup: tiles t with t % 2 == sg
    const int q4 = warp & 3;                 // tensor-memory lane quarter of this warp
    const int st = tid - 64;                 // 0..255 within the softmax warps
    const int lrow = q4 * 32 + lane;         // tile position (S) or d (O) of this thread
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const float scale = p.scale, scale2 = p.scale * kLog2e;
    const int swz_row = (NP == 16) ? ((lrow >> 2) & 1) : ((lrow >> 1) & 3);

    // record of chunk m: O^T buffer m&1 -> workspace, with its row max / sum from cm / cl
    auto epilogue = [&](int m) -> bool {
      const Item x = make_item<NP>(blockIdx.x + m * gridDim.x, pref, lens_s, rid_s, batch, p);
      if (!wait_bar(smem_u32(&B->o_full[m & 1]), (m >> 1) & 1, abort_flag, p.err)) return false;
      tc_fence_after();
      const size_t rec_floats = (size_t)p.Rp * (kD + 2);
      float* rec = p.part + (((size_t)x.r * Hkv + x.kvh) * p.nchunk_max + x.c) * rec_floats;
      constexpr int kHalf = NP / 2 >= 16 ? NP / 2 : 16;    // columns per warpgroup
      if (sg * kHalf < NP) {
        float o[16];
        tmem_ld16(tl + C::kOCol + (m & 1) * NP + sg * kHalf, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) rec[2 * p.Rp + (size_t)(sg * kHalf + j) * kD + lrow] = o[j];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&B->o_empty[m & 1]));
      if (st < NP) {
        rec[st] = cm[(m & 1) * NP + st];
        rec[p.Rp + st] = cl[(m & 1) * NP + st];
      }
      return true;
    };

    bool ok = true;
    for (int n = 0; n < my_items && !aborted(abort_flag); ++n) {
      const Item x = make_item<NP>(blockIdx.x + n * gridDim.x, pref, lens_s, rid_s, batch, p);
      const int L = x.L, start = x.start, end = x.end;
      float* scores = p.scores ? p.scores + ((size_t)x.r * Hkv + x.kvh) * (size_t)p.cap * R : nullptr;
      if (!wait_bar(smem_u32(&B->s_full[n & 1]), (n >> 1) & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sbuf = tl + (n & 1) * C::kSCols;

      // pass 1 over this warpgroup's tiles: committed logits out, max per row (raw units)
      float mrow[NP];
#pragma unroll
      for (int j = 0; j < NP; ++j) mrow[j] = -INFINITY;
      for (int t = sg; t < x.ntile; t += 2) {
        float v[NP];
        tmem_ld<NP>(sbuf + t * NP, v);
        tmem_wait_ld();
        const int t0 = start + t * kPos;
        const int pos = t0 + lrow;
        if (scores && pos < L) {
          float* dst = scores + (size_t)pos * R;
          if ((R & 3) == 0) {
#pragma unroll
            for (int j = 0; j < NP; j += 4)
              if (j < R)
                *reinterpret_cast<float4*>(dst + j) =
                    make_float4(v[j] * scale, v[j + 1] * scale, v[j + 2] * scale, v[j + 3] * scale);
          } else {
#pragma unroll
            for (int j = 0; j < NP; ++j)
              if (j < R) dst[j] = v[j] * scale;
          }
        }
        if (t0 + kPos <= min(L, end)) {
#pragma unroll
          for (int j = 0; j < NP; ++j) mrow[j] = fmaxf(mrow[j], v[j]);
        } else {
#pragma unroll
          for (int j = 0; j < NP; ++j) {
            const bool vis = pos < end && j < R && (pos < L || pos - L <= trow[j]);
            if (vis) mrow[j] = fmaxf(mrow[j], v[j]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        float m = mrow[j];
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
        if (lane == j) redM[sw8 * NP + j] = m;
      }
      named_sync_softmax();
      if (st < NP) {
        float m = redM[st];
#pragma unroll
        for (int w = 1; w < 8; ++w) m = fmaxf(m, redM[w * NP + st]);
        cm[(n & 1) * NP + st] = scale2 * m;
      }
      named_sync_softmax();
#pragma unroll
      for (int j = 0; j < NP; ++j) mrow[j] = cm[(n & 1) * NP + j];

      // the previous chunk's output leaves tensor memory before P^T is overwritten
      if (n > 0 && !epilogue(n - 1)) {
        ok = false;
        break;
      }

      // pass 2: P = 2^(s - max) as bf16 P^T tiles (MN-major, NP values per position) + sums
      float lsum[NP];
#pragma unroll
      for (int j = 0; j < NP; ++j) lsum[j] = 0.f;
      for (int t = sg; t < x.ntile; t += 2) {
        float v[NP];
        tmem_ld<NP>(sbuf + t * NP, v);
        tmem_wait_ld();
        const int t0 = start + t * kPos;
        const int pos = t0 + lrow;
        const bool interior = t0 + kPos <= min(L, end);
        uint32_t pk[NP / 2];
#pragma unroll
        for (int j = 0; j < NP; j += 2) {
          float e0 = ex2(fmaf(v[j], scale2, -mrow[j]));
          float e1 = ex2(fmaf(v[j + 1], scale2, -mrow[j + 1]));
          if (!interior) {
            const bool v0 = pos < end && j < R && (pos < L || pos - L <= trow[j]) && mrow[j] != -INFINITY;
            const bool v1 = pos < end && j + 1 < R && (pos < L || pos - L <= trow[j + 1]) &&
                            mrow[j + 1] != -INFINITY;
            e0 = v0 ? e0 : 0.f;
            e1 = v1 ? e1 : 0.f;
          }
          lsum[j] += e0;
          lsum[j + 1] += e1;
          pk[j / 2] = pack_bf16(e0, e1);
        }
        uint8_t* prow = smem + C::kPOff + t * C::kPTile + lrow * (NP * 2);
#pragma unroll
        for (int cc = 0; cc < NP / 8; ++cc)
          *reinterpret_cast<uint4*>(prow + ((cc ^ swz_row) << 4)) =
              make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      }
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&B->s_empty[n & 1]));
        mbar_arrive(smem_u32(&B->p_full));
      }
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        float sacc = lsum[j];
#pragma unroll
        for (int o = 16; o; o >>= 1) sacc += __shfl_xor_sync(kFull, sacc, o);
        if (lane == j) redL[sw8 * NP + j] = sacc;
      }
      named_sync_softmax();
      if (st < NP) {
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) l += redL[w * NP + st];
        cl[(n & 1) * NP + st] = l;
      }
      // (cl / redL reuse is ordered by the barriers of the next chunk)
    }
    if (ok && my_items > 0 && !aborted(abort_flag)) {
      named_sync_softmax();   // cl of the last chunk complete
      epilogue(my_items - 1);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace tc

int verify_tc_npad(int R) { return R <= 16 ? 16 : (R <= 32 ? 32 : 0); }

template <int NP>
static int launch_tc(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tk8,
                     const CUtensorMap& tv8, const VerifyParams& p, int batch, int num_sms,
                     cudaStream_t stream) {
  using C = tc::Cfg<NP>;
  static bool attr_done = false;
  if (!attr_done) {
    if (cuda_status(cudaFuncSetAttribute(tc::verify_tc_kernel<NP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem),
                    "cudaFuncSetAttribute") != S3R_OK)
      return S3R_ERR_CUDA;
    attr_done = true;
  }
  tc::verify_tc_kernel<NP><<<num_sms, tc::kThreads, C::kSmem, stream>>>(tk, tv, tk8, tv8, p, batch);
  return cuda_status(cudaGetLastError(), __func__);
}

bool verify_tc_supported(int D, int R, int batch) {
  return D == tc::kD && verify_tc_npad(R) != 0 && batch <= tc::kMaxBatch;
}

int verify_tc_chunk(int R) {
  const int np = verify_tc_npad(R);
  return np == 16 ? tc::Cfg<16>::kChunk : tc::Cfg<32>::kChunk;
}

int launch_verify_tc(const CUtensorMap& k1, const CUtensorMap& v1, const CUtensorMap& k8,
                     const CUtensorMap& v8, const VerifyParams& p, int batch, int num_sms,
                     cudaStream_t stream) {
  const int np = verify_tc_npad(p.R);
  if (np == 16) return launch_tc<16>(k1, v1, k8, v8, p, batch, num_sms, stream);
  if (np == 32) return launch_tc<32>(k1, v1, k8, v8, p, batch, num_sms, stream);
  return S3R_ERR_UNSUPPORTED;
}

}  // namespace s3r
