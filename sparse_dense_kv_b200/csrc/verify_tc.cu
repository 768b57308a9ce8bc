// Dense verify attention with score capture on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory), head_dim 128, up to 64 rows per KV head (padded to 16, 32,
// 48 or 64 rows: N of both products).
//
// What it computes is what verify.cu computes ([News] Interpretation: the proposed block is
// recomputed against the complete historical KV; [Explainer] walkthrough: the sparse set
// comes from the verifier's last attention pass): rows (t, g) at positions L+t attend
// positions 0..L+t; out, lse and every committed logit are written.
//
// Organisation (one persistent CTA per SM, 12 warps). A work item is (request, KV head,
// chunk of up to 8, 7, 4 or 3 tiles of 128 positions at 16, 32, 48 or 64 rows: two S
// buffers of a chunk and two O buffers fill the 512 columns of tensor memory). Items are
// claimed from a counter in the workspace as CTAs progress (the K producer claims, a ring in
// shared memory tells the other roles), so faster SMs take more of them.
//   warp 0     K producer: per item it loads the item's Q rows into one of two Q buffers
//              (3-D TMA box, rows t*G+g), then streams the chunk's K tiles through a
//              2-stage ring with 4-D TMA over (d, slot, head, page): a tile of 8
//              consecutive page ids is 2 boxes (one per 64-column half, 128-byte swizzle),
//              otherwise one box per page and half. The tile holding the block (positions
//              >= L) is patched after its TMA lands. It also writes the block into the cache.
//              The next item is claimed, and its page ids and Q rows fetched, once the
//              current item's first tile is on its way.
//   warp 1     V producer: the same for the V tiles, through its own 2-stage ring, so the
//              K stream of item n+1 and the V stream of item n run side by side.
//   warp 2     QK issuer: S^T tile t (128 positions x N rows, fp32) = K_t . Q^T into tensor
//              memory, item after item. K and Q are K-major operands (128-byte swizzle).
//   warp 11    PV issuer: O^T (128 d x N) += V_t^T . P_t^T, item after item, once the item's
//              P^T is written. V^T is MN-major (the V tile as it arrives) and so is P^T (N
//              values per position in atoms of 16, 32 or 64 rows: 32-, 64- or 128-byte
//              swizzle; 48 rows are three 16-row atoms). S and O are double-buffered in
//              tensor memory. The two issuers block on their own barriers, so neither
//              product waits for the other's issue (each tile's eight dependent MMAs take
//              about half a microsecond to issue).
//   warps 3-10 softmax / epilogue, two warpgroups each owning half of the rows (one thread
//              per tensor-memory lane = position or d): pass 1 reads every S tile, writes the
//              committed logits and takes the chunk maximum per row; pass 2 re-reads them and
//              writes P = 2^(s - max) as bf16 P^T tiles. P^T is single-buffered: a tile is
//              rewritten for item n+1 once the PV of item n has read it (a barrier per
//              tile), so that PV and pass 2 of item n+1 overlap; the PV of an item starts
//              once its whole P^T is written. Then the chunk record (max, sum, O) goes to the
//              workspace, and a second kernel merges the chunks of every (request, KV head).
// Every wait is bounded (an expired wait sets S3R_ERR_TIMEOUT and the CTA winds down).
// The softmax is exact per chunk (two passes over logits resident in tensor memory), so no
// running rescale exists; chunks merge by their (max, sum) as in the CUDA-core kernel.
#include "attention.cuh"
#include "kernels.h"

namespace s3r {
namespace tc {

constexpr int kPos = 128;                   // positions per tile (MMA M)
constexpr int kD = 128;                     // head_dim of this path
constexpr int kMaxStages = 4;               // ring barriers per stream
constexpr int kThreads = 384;               // K producer, V producer, QK MMA, 8 softmax, PV MMA warps
constexpr int kSoftWarp0 = 3;
constexpr int kPvWarp = 11;
constexpr int kBarBytes = 768;              // mbarriers and flags
constexpr int kRing = 16;                   // item ids published by the K producer
constexpr int kTileBytes = kPos * kD * 2;   // 32 KB: [2 halves][128 rows][128 B]
constexpr int kMaxBatch = 256;              // requests per launch (larger batches: several launches)

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
// This warp's 32 lanes x 8 consecutive columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
// N (a multiple of 8) consecutive columns in loads of 16 and, if N % 16 == 8, one of 8.
// Every 16-column load starts on a multiple of 16 columns: lead8 says the first column is
// 8 past one (the upper half of 48 rows starts at column 24), so the 8-column load goes first.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[N], bool lead8 = false) {
  static_assert(N % 8 == 0, "whole groups of 8 columns");
  auto run16 = [&](int first) {
#pragma unroll
    for (int c = first; c + 16 <= N; c += 16) {
      float w[16];
      tmem_ld16(taddr + c, w);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[c + i] = w[i];
    }
  };
  if constexpr (N % 16 == 8) {
    if (lead8) {
      tmem_ld8(taddr, v);
      run16(8);
    } else {
      run16(0);
      tmem_ld8(taddr + (N - 8), v + (N - 8));
    }
  } else {
    run16(0);
  }
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
  static constexpr int kTiles = NP == 64 ? 3 : (NP == 48 ? 4 : (NP == 32 ? 7 : 8));   // tiles per chunk
  static constexpr int kKSt = 2;                             // K ring stages
  static constexpr int kVSt = 2;                             // V ring stages
  static constexpr int kChunk = kTiles * kPos;
  static constexpr int kQBytes = 2 * NP * 128;               // one Q buffer: [2 halves][NP rows][128 B]
  static constexpr int kPTile = kPos * NP * 2;               // P^T tile: [128 pos][NP rows] bf16
  static constexpr int kPBytes = kTiles * kPTile;
  // P^T swizzle: 32 bytes for 16 and 48 rows (one or three 16-row atoms along N), 64 for
  // 32, 128 for 64 (one atom)
  static constexpr uint32_t kPSwz = (NP == 16 || NP == 48) ? 6u : (NP == 32 ? 4u : 2u);
  static constexpr int kPAtomRows = (NP == 16 || NP == 48) ? 16 : NP;       // rows of one atom
  static constexpr int kPAtomBytes = kPos * kPAtomRows * 2;                 // one atom column of a tile
  static constexpr int kTmemCols = 512;
  static constexpr int kSCols = kTiles * NP;                 // one S buffer
  static constexpr int kOCol = 2 * kSCols;                   // two O buffers after two S buffers
  static_assert(kOCol + 2 * NP <= kTmemCols, "tensor memory budget");
  static_assert(kKSt <= kMaxStages && kVSt <= kMaxStages && kTiles <= 8, "barrier arrays");
  static constexpr int kSmemMax = 227 * 1024;
  static constexpr int kKRingOff = 0;
  static constexpr int kVRingOff = kKSt * kTileBytes;
  static constexpr int kQOff = (kKSt + kVSt) * kTileBytes;
  static constexpr int kPOff = kQOff + 2 * kQBytes;         // two Q buffers (item parity)
  static constexpr int kRedOff = kPOff + kPBytes;            // redM, redL [8 warps][NP]; cm, cl [2][NP]
  static constexpr int kRedBytes = (2 * 8 * NP + 4 * NP) * 4;
  static constexpr int kPrefOff = kRedOff + kRedBytes;       // request prefix [kMaxBatch+1]
  static constexpr int kLenOff = kPrefOff + (kMaxBatch + 1) * 4;   // L per request [kMaxBatch]
  static constexpr int kRidOff = kLenOff + kMaxBatch * 4;          // request id [kMaxBatch]
  static constexpr int kIdsOff = kRidOff + kMaxBatch * 4;          // page ids [K, V producer][64]
  static constexpr int kBarOff = (kIdsOff + 2 * 64 * 4 + 63) / 64 * 64;
  static constexpr int kSmem = kBarOff + kBarBytes + 1024;   // + barriers + alignment slack
  static_assert(kSmem <= kSmemMax, "shared memory budget");
  static_assert(kQOff % 1024 == 0 && kPOff % 1024 == 0 && kRedOff % 16 == 0 && kBarOff % 64 == 0,
                "alignment of the swizzled operands, the reduction scratch and the barriers");
};

struct Bars {
  uint64_t kfull[kMaxStages], kempty[kMaxStages], ktma[kMaxStages];
  uint64_t vfull[kMaxStages], vempty[kMaxStages], vtma[kMaxStages];
  // one barrier pair per tensor-memory buffer (chunk parity), so that no barrier ever runs
  // two phases ahead of a waiter
  uint64_t q_full[2], q_empty[2], p_full, fin[2];
  uint64_t s_full[2], s_empty[2], o_full[2], o_empty[2];
  uint64_t p_free[8];   // P^T tile t has been read by the PV of the previous chunk
  uint64_t wg[2];       // barrier of each softmax warpgroup (4 warps)
  uint64_t item_bar[kRing];   // item id of the CTA's m-th item published in item_id[m % kRing]
  int item_id[kRing];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= kBarBytes, "barrier block");



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
    verify_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmK8, const __grid_constant__ CUtensorMap tmV8,
                     const VerifyParams p, int batch) {
  pdl_wait();
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
  const int T = p.T, G = p.G, R = p.R, Hkv = p.Hkv;
  const int chunk = C::kChunk;
  const uint32_t sbase = smem_u32(smem);

  // ---- set-up: request prefix (items), barriers, tensor memory
  for (int b = tid; b < batch; b += blockDim.x) {
    const int r = p.req_ids ? p.req_ids[p.req_off + b] : p.req_off + b;
    const bool known = r >= 0 && r < p.num_requests;   // else no items, bounds reported
    const int L = known ? p.seq_lens[r] : -1;
    const int Lc = L + T;
    rid_s[b] = known ? r : 0;
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
    for (int s = 0; s < C::kKSt; ++s) {
      mbar_init(smem_u32(&B->kfull[s]), 1);
      mbar_init(smem_u32(&B->kempty[s]), 1);
      mbar_init(smem_u32(&B->ktma[s]), 1);
    }
    for (int s = 0; s < C::kVSt; ++s) {
      mbar_init(smem_u32(&B->vfull[s]), 1);
      mbar_init(smem_u32(&B->vempty[s]), 1);
      mbar_init(smem_u32(&B->vtma[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&B->q_full[b]), 1);
      mbar_init(smem_u32(&B->q_empty[b]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&B->s_full[b]), 1);
      mbar_init(smem_u32(&B->s_empty[b]), 8);
      mbar_init(smem_u32(&B->o_full[b]), 1);
      mbar_init(smem_u32(&B->o_empty[b]), 8);
    }
    mbar_init(smem_u32(&B->p_full), 8);
    for (int t = 0; t < 8; ++t) mbar_init(smem_u32(&B->p_free[t]), 1);
    for (int i = 0; i < kRing; ++i) mbar_init(smem_u32(&B->item_bar[i]), 1);
    mbar_init(smem_u32(&B->wg[0]), 4);
    mbar_init(smem_u32(&B->wg[1]), 4);
    mbar_init(smem_u32(&B->fin[0]), 1);
    mbar_init(smem_u32(&B->fin[1]), 1);
    B->abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&B->tmem_base), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;
  const int nitems = pref[batch];
  // Work is claimed, not dealt: a CTA's first item is blockIdx.x, every later one comes from
  // the launch's counter (item gridDim.x + counter), claimed by the K producer one item
  // ahead of its own progress and published in the ring (item id nitems: no more work), so
  // CTAs on faster SMs take more chunks and all finish within about one chunk of each other.
  auto ring_id = [&](int m) -> int {   // warp-uniform; -1 if the wait gave up
    const int slot = m & (kRing - 1);
    if (!wait_bar(smem_u32(&B->item_bar[slot]), (uint32_t)(m / kRing) & 1u, abort_flag, p.err, p.wait_limit)) return -1;
    return *reinterpret_cast<volatile int*>(&B->item_id[slot]);
  };
  const uint32_t qbuf = sbase + C::kQOff, pbuf = sbase + C::kPOff;

  if (warp <= 1) {
    // ============================================================ producers ====
    // warp 0 streams the K tiles of every item (and its Q rows), warp 1 the V tiles, each
    // through its own ring, so the two streams never wait on each other
    const bool is_v = warp == 1;
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(is_v ? &tmV : &tmK)) : "memory");
      asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(is_v ? &tmV8 : &tmK8)) : "memory");
      if (!is_v) asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tmQ)) : "memory");
    }
    const int nst = is_v ? C::kVSt : C::kKSt;
    const int roff = is_v ? C::kVRingOff : C::kKRingOff;
    uint64_t* full = is_v ? B->vfull : B->kfull;
    uint64_t* empty = is_v ? B->vempty : B->kempty;
    uint64_t* tmab = is_v ? B->vtma : B->ktma;
    const CUtensorMap* map = is_v ? &tmV : &tmK;
    const CUtensorMap* map8 = is_v ? &tmV8 : &tmK8;
    const __nv_bfloat16* blk = is_v ? p.v_new : p.k_new;
    int* ids_own = ids_s + (is_v ? 64 : 0);
    int g = 0;
    uint32_t tma_phase = 0;   // bit s: phase of tma[s]
    bool stop = false;
    // after_first() runs once, when the item's first tile is on its way
    auto load_tiles = [&](const Item& x, auto&& after_first) {
      for (int t = 0; t < x.ntile && !stop; ++t, ++g) {
        const int s = g % nst;
        if (g >= nst && !wait_bar(smem_u32(&empty[s]), ((g / nst) - 1) & 1, abort_flag, p.err, p.wait_limit)) {
          stop = true;
          break;
        }
        const int t0 = x.start + t * kPos;
        const uint32_t dst = sbase + roff + s * kTileBytes;
        uint32_t okmask = 0;
        int nload = 0;
        bool tail = (t0 + kPos > x.L);
        int ids[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) ids[i] = ids_own[t * 8 + i];
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
        const uint32_t landing = smem_u32(tail ? &tmab[s] : &full[s]);
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
          if (!wait_bar(smem_u32(&tmab[s]), (tma_phase >> s) & 1, abort_flag, p.err, p.wait_limit)) {
            mbar_wait(smem_u32(&tmab[s]), (tma_phase >> s) & 1);   // its copies land before exit
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
            *reinterpret_cast<uint4*>(smem + roff + s * kTileBytes + off) = v;
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&full[s]));
        }
        __syncwarp();
        if (t == 0) after_first();
      }
    };
    if (!is_v) {
      // Q padding rows R..NP-1 of both halves of both buffers stay zero: the Q copies
      // write rows < R only
      for (int idx = lane; idx < 4 * (NP - R) * 8; idx += 32) {
        const int h = idx / ((NP - R) * 8), rem = idx - h * (NP - R) * 8;   // h: buffer*2 + half
        *reinterpret_cast<uint4*>(smem + C::kQOff + h * (NP * 128) + (R + (rem >> 3)) * 128 +
                                  ((rem & 7) << 4)) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async();
      __syncwarp();
    }
    // page ids of an item's committed pages (-1 past L), two per lane, loaded one item ahead
    auto fetch_ids = [&](const Item& x, int& a, int& b) {
      const int* ptab = p.page_table + (size_t)x.r * p.max_pages;
      const int npg = x.ntile * 8;
      const int pg0 = x.start >> 4;
      a = lane < npg && (pg0 + lane) * kPage < x.L ? ptab[pg0 + lane] : -1;
      b = lane + 32 < npg && (pg0 + lane + 32) * kPage < x.L ? ptab[pg0 + lane + 32] : -1;
    };
    // id of the CTA's m-th item: the K producer claims and publishes it, the V producer
    // reads it from the ring
    auto item_id = [&](int m) -> int {
      if (is_v) return ring_id(m);
      int id = (int)blockIdx.x;
      if (m > 0) {
        int v = 0;
        if (lane == 0) v = atomicAdd(p.sched, 1);
        id = __shfl_sync(kFull, v, 0) + (int)gridDim.x;
      }
      id = min(id, nitems);
      if (lane == 0) {
        B->item_id[m & (kRing - 1)] = id;
        mbar_arrive(smem_u32(&B->item_bar[m & (kRing - 1)]));   // release: the id is visible
      }
      __syncwarp();
      return id;
    };
    int q_issued = 0;   // Q loads issued (item m's load lands on q_full[m & 1], phase (m >> 1) & 1)
    // K producer: item m's Q rows -> Q buffer m&1 by TMA (K-major, 128-byte swizzle) once the
    // QK of item m-2 has read that buffer
    auto load_q = [&](const Item& x, int m) -> bool {
      const int qb = m & 1;
      if (m >= 2 && !wait_bar(smem_u32(&B->q_empty[qb]), ((m - 2) >> 1) & 1, abort_flag, p.err, p.wait_limit))
        return false;
      if (lane == 0) mbar_arrive_expect_tx(smem_u32(&B->q_full[qb]), (uint32_t)(2 * R * 128));
      __syncwarp();
      if (lane < 2)
        tma_load_3d(qbuf + qb * C::kQBytes + lane * (NP * 128), &tmQ, lane * 64, x.kvh * G, x.r * T,
                    smem_u32(&B->q_full[qb]));
      q_issued = m + 1;
      __syncwarp();
      return true;
    };
    int cur = item_id(0);
    Item x{};
    int ida = -1, idb = -1;   // page ids of item m (two per lane)
    if (cur >= 0 && cur < nitems) {
      x = make_item<NP>(cur, pref, lens_s, rid_s, batch, p);
      fetch_ids(x, ida, idb);
      if (!is_v && !load_q(x, 0)) stop = true;
    }
    for (int m = 0; cur >= 0 && cur < nitems && !stop && !aborted(abort_flag); ++m) {
      __syncwarp();   // every lane is done with the previous item's ids
      ids_own[lane] = ida;
      ids_own[lane + 32] = idb;
      __syncwarp();
      // The next item is claimed (K) or read from the ring (V), its page ids fetched and its
      // Q rows loaded (K) once this item's first tile is on its way, so those round trips
      // overlap the ring's waits instead of leaving the stream idle between items.
      int nxt = -1, na = -1, nb = -1;
      Item xn{};
      bool ahead = false;
      auto next_item = [&]() {
        ahead = true;
        nxt = item_id(m + 1);
        if (nxt >= 0 && nxt < nitems) {
          xn = make_item<NP>(nxt, pref, lens_s, rid_s, batch, p);
          fetch_ids(xn, na, nb);
          if (!is_v && !load_q(xn, m + 1)) stop = true;
        }
      };
      load_tiles(x, next_item);
      if (!ahead && !stop) next_item();
      if (!is_v && x.c == 0 && !stop) {   // the block's K/V enter the cache once per (request, head)
        const int* ptab = p.page_table + (size_t)x.r * p.max_pages;
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
      cur = nxt;
      x = xn;
      ida = na;
      idb = nb;
    }
    // nothing may still be landing in this ring (or a Q buffer) when the CTA exits, also after
    // an abort: these waits are for this warp's own copies and are not cut short
    for (int q = g - nst > 0 ? g - nst : 0; q < g; ++q) mbar_wait(smem_u32(&full[q % nst]), (q / nst) & 1);
    for (int m = q_issued - 2 > 0 ? q_issued - 2 : 0; m < q_issued; ++m)
      mbar_wait(smem_u32(&B->q_full[m & 1]), (uint32_t)(m >> 1) & 1u);
  } else if (warp == 2 || warp == kPvWarp) {
    // ===================================================================== MMA warps ===
    // Warp 2 issues the QK products of the CTA's items in order (S^T = K_t . Q^T per tile,
    // once the tile, the item's Q rows and a free S buffer are there); warp kPvWarp issues
    // the PV products (O^T += V_t^T . P_t^T, once the softmax has written the item's P^T and
    // its O buffer is free). Each blocks on its own barriers, so a PV never waits for the
    // issue of QK tiles of a later item, nor the reverse.
    const bool is_pv = warp == kPvWarp;
    constexpr uint32_t kIdQK = idesc_bf16(kPos, NP, false, false);
    constexpr uint32_t kIdPV = idesc_bf16(kD, NP, true, true);
    if (!is_pv) {
      int gk = 0;
      for (int mk = 0;; ++mk) {
        const int id = ring_id(mk);
        if (id < 0 || id >= nitems) break;
        const Item xk = make_item<NP>(id, pref, lens_s, rid_s, batch, p);
        if (!wait_bar(smem_u32(&B->q_full[mk & 1]), (mk >> 1) & 1, abort_flag, p.err, p.wait_limit)) break;
        if (mk >= 2 &&
            !wait_bar(smem_u32(&B->s_empty[mk & 1]), ((mk - 2) >> 1) & 1, abort_flag, p.err, p.wait_limit))
          break;
        bool ok = true;
        for (int tk = 0; tk < xk.ntile; ++tk, ++gk) {
          const int s = gk % C::kKSt;
          if (!wait_bar(smem_u32(&B->kfull[s]), (gk / C::kKSt) & 1, abort_flag, p.err, p.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t kt = sbase + C::kKRingOff + s * kTileBytes;
            const uint32_t sd = tmem + (mk & 1) * C::kSCols + tk * NP;
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint64_t ad = sdesc(kt + (kk >> 2) * (kPos * 128) + (kk & 3) * 32, 16, 1024, 2);
              const uint64_t bd = sdesc(qbuf + (mk & 1) * C::kQBytes + (kk >> 2) * (NP * 128) +
                                            (kk & 3) * 32, 16, 1024, 2);
              tc_mma(sd, ad, bd, kIdQK, kk > 0 ? 1u : 0u);
            }
            tc_commit(smem_u32(&B->kempty[s]));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) {
          tc_commit(smem_u32(&B->s_full[mk & 1]));
          tc_commit(smem_u32(&B->q_empty[mk & 1]));
        }
        __syncwarp();
      }
    } else {
      int gv = 0;
      for (int nv = 0;; ++nv) {
        const int id = ring_id(nv);
        if (id < 0 || id >= nitems) break;
        const Item xv = make_item<NP>(id, pref, lens_s, rid_s, batch, p);
        if (!wait_bar(smem_u32(&B->p_full), nv & 1, abort_flag, p.err, p.wait_limit)) break;
        if (nv >= 2 &&
            !wait_bar(smem_u32(&B->o_empty[nv & 1]), ((nv - 2) >> 1) & 1, abort_flag, p.err, p.wait_limit))
          break;
        bool ok = true;
        for (int tv = 0; tv < xv.ntile; ++tv, ++gv) {
          const int s = gv % C::kVSt;
          if (!wait_bar(smem_u32(&B->vfull[s]), (gv / C::kVSt) & 1, abort_flag, p.err, p.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t vt = sbase + C::kVRingOff + s * kTileBytes;
            const uint32_t pt = pbuf + tv * C::kPTile;
            const uint32_t od = tmem + C::kOCol + (nv & 1) * NP;
#pragma unroll
            for (int kk = 0; kk < kPos / 16; ++kk) {
              const uint64_t ad = sdesc(vt + kk * 2048, kPos * 128, 1024, 2);
              // MN-major P^T: LBO = stride between atoms along N, SBO = stride between
              // groups of 8 positions (one atom row is kPAtomRows * 2 bytes)
              const uint64_t bd = sdesc(pt + kk * 16 * C::kPAtomRows * 2, C::kPAtomBytes,
                                        8 * C::kPAtomRows * 2, C::kPSwz);
              tc_mma(od, ad, bd, kIdPV, (tv > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(smem_u32(&B->vempty[s]));
            tc_commit(smem_u32(&B->p_free[tv]));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) {
          // every P^T tile's barrier completes once per chunk, used or not
          for (int t = xv.ntile; t < C::kTiles; ++t) tc_commit(smem_u32(&B->p_free[t]));
          tc_commit(smem_u32(&B->o_full[nv & 1]));
        }
        __syncwarp();
      }
    }
    // make sure nothing this warp issued is still running before the tensor memory goes away
    if (lane == 0) tc_commit(smem_u32(&B->fin[is_pv ? 1 : 0]));
    __syncwarp();
    mbar_wait(smem_u32(&B->fin[is_pv ? 1 : 0]), 0);   // not cut short by an abort: the work is in flight
  } else {
    // ================================================================ softmax warps ===
    // Warpgroup sg owns rows (columns of S and O^T) [sg*NH, sg*NH + NH) of every tile; the
    // two warpgroups only meet at the chunk's barriers for the MMA warps.
    constexpr int NH = NP / 2;               // rows per warpgroup
    // tiles per tensor-memory wait: one from 32 rows up (two tiles' values in flight made the
    // 32-row pass 2 twice as slow, measured), four at 16
    constexpr int BT = NP >= 32 ? 1 : 4;
    const int sw8 = warp - kSoftWarp0;       // 0..7
    const int sg = sw8 >> 2;                 // warpgroup
    const int sw4 = sw8 & 3;                 // warp within the warpgroup
    const int q4 = warp & 3;                 // tensor-memory lane quarter of this warp
    const int gt = (tid - 32 * kSoftWarp0) & 127;   // thread within the warpgroup
    const int lrow = q4 * 32 + lane;         // tile position (S) or d (O) of this thread
    const int c0 = sg * NH;                  // first row of this warpgroup
    const bool lead8 = (c0 & 15) == 8;       // its columns start 8 past a multiple of 16
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const float scale = p.scale, scale2 = p.scale * kLog2e;
    // the row's 16-byte chunk is XORed with address bits 7.. of its P^T row (32-, 64-, 128-byte swizzle)
    const int swz_row = (NP == 16 || NP == 48) ? ((lrow >> 2) & 1) : (NP == 32 ? ((lrow >> 1) & 3) : (lrow & 7));
    // Warpgroup barrier on an mbarrier (bounded wait, unlike bar.sync): if a wait anywhere
    // gives up, the other warps of the group give up here too instead of hanging.
    uint32_t wg_phase = 0;
    auto wg_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&B->wg[sg]));
      const bool r = wait_bar(smem_u32(&B->wg[sg]), wg_phase, abort_flag, p.err, p.wait_limit);
      wg_phase ^= 1u;
      return r;
    };

    // record of chunk m (this warpgroup's rows): O^T buffer m&1 -> workspace, with the rows'
    // max / sum from cm / cl
    auto epilogue = [&](int m, const Item& x) -> bool {
      if (!wait_bar(smem_u32(&B->o_full[m & 1]), (m >> 1) & 1, abort_flag, p.err, p.wait_limit)) return false;
      tc_fence_after();
      const size_t rec_floats = (size_t)p.Rp * (kD + 2);
      float* rec = p.part + (((size_t)x.r * Hkv + x.kvh) * p.nchunk_max + x.c) * rec_floats;
      float o[NH];
      tmem_ld_cols<NH>(tl + C::kOCol + (m & 1) * NP + c0, o, lead8);
      tmem_wait_ld();
      // records hold the R real rows (row pitch p.Rp >= R)
#pragma unroll
      for (int j = 0; j < NH; ++j)
        if (c0 + j < R) rec[2 * p.Rp + (size_t)(c0 + j) * kD + lrow] = o[j];
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&B->o_empty[m & 1]));
      if (gt < NH && c0 + gt < R) {
        rec[c0 + gt] = cm[(m & 1) * NP + c0 + gt];
        rec[p.Rp + c0 + gt] = cl[(m & 1) * NP + c0 + gt];
      }
      return true;
    };

    bool ok = true;
    int n = 0;
    Item xprev{};
    for (; !aborted(abort_flag); ++n) {
      const int id = ring_id(n);
      if (id < 0) {
        ok = false;
        break;
      }
      if (id >= nitems) break;
      const Item x = make_item<NP>(id, pref, lens_s, rid_s, batch, p);
      const int L = x.L, start = x.start, end = x.end;
      float* scores = p.scores ? p.scores + ((size_t)x.r * Hkv + x.kvh) * (size_t)R * p.cap : nullptr;
      if (!wait_bar(smem_u32(&B->s_full[n & 1]), (n >> 1) & 1, abort_flag, p.err, p.wait_limit)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sbuf = tl + (n & 1) * C::kSCols + c0;

      // pass 1 over every tile: committed logits out, max per row (raw units)
      float mrow[NH];
#pragma unroll
      for (int j = 0; j < NH; ++j) mrow[j] = -INFINITY;
      for (int tb = 0; tb < x.ntile; tb += BT) {
        float vv[BT][NH];
#pragma unroll
        for (int u = 0; u < BT; ++u)   // past the last tile: reload the last tile (unused)
          tmem_ld_cols<NH>(sbuf + min(tb + u, x.ntile - 1) * NP, vv[u], lead8);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < BT; ++u) {
          if (tb + u >= x.ntile) break;
          const int t0 = start + (tb + u) * kPos;
          const int pos = t0 + lrow;
          if (scores && pos < L) {
            // committed logits, [row][position]: the warp's 32 lanes write 32 consecutive
            // positions of one row per store, one whole 128-byte line
#pragma unroll
            for (int j = 0; j < NH; ++j)
              if (c0 + j < R) scores[(size_t)(c0 + j) * p.cap + pos] = vv[u][j] * scale;
          }
          if (t0 + kPos <= min(L, end)) {
#pragma unroll
            for (int j = 0; j < NH; ++j) mrow[j] = fmaxf(mrow[j], vv[u][j]);
          } else {
#pragma unroll
            for (int j = 0; j < NH; ++j) {
              const int row = c0 + j;
              const bool vis = pos < end && row < R && (pos < L || pos - L <= trow[row]);
              if (vis) mrow[j] = fmaxf(mrow[j], vv[u][j]);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < NH; ++j) {
        float m = mrow[j];
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
        if (lane == j) redM[(sg * 4 + sw4) * NH + j] = m;
      }
      if (!wg_sync()) {
        ok = false;
        break;
      }
      if (gt < NH) {
        float m = redM[(sg * 4) * NH + gt];
#pragma unroll
        for (int w = 1; w < 4; ++w) m = fmaxf(m, redM[(sg * 4 + w) * NH + gt]);
        cm[(n & 1) * NP + c0 + gt] = scale2 * m;
      }
      if (!wg_sync()) {
        ok = false;
        break;
      }
#pragma unroll
      for (int j = 0; j < NH; ++j) mrow[j] = cm[(n & 1) * NP + c0 + j];

      // pass 2: P = 2^(s - max) as bf16 P^T tiles (MN-major, NP values per position; this
      // warpgroup writes its NH of them) + sums. P^T tile t is overwritten once the previous
      // chunk's PV has read it (its own barrier), so this pass runs alongside that PV.
      float lsum[NH];
#pragma unroll
      for (int j = 0; j < NH; ++j) lsum[j] = 0.f;
      for (int tb = 0; tb < x.ntile && ok; tb += BT) {
        float vv[BT][NH];
#pragma unroll
        for (int u = 0; u < BT; ++u)   // past the last tile: reload the last tile (unused)
          tmem_ld_cols<NH>(sbuf + min(tb + u, x.ntile - 1) * NP, vv[u], lead8);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < BT; ++u) {
          if (tb + u >= x.ntile) break;
          const int t = tb + u;
          const int t0 = start + t * kPos;
          const int pos = t0 + lrow;
          const bool interior = t0 + kPos <= min(L, end);
          uint32_t pk[NH / 2];
#pragma unroll
          for (int j = 0; j < NH; j += 2) {
            float e0 = ex2(fmaf(vv[u][j], scale2, -mrow[j]));
            float e1 = ex2(fmaf(vv[u][j + 1], scale2, -mrow[j + 1]));
            if (!interior) {
              const int r0 = c0 + j, r1 = c0 + j + 1;
              const bool v0 = pos < end && r0 < R && (pos < L || pos - L <= trow[r0]) && mrow[j] != -INFINITY;
              const bool v1 = pos < end && r1 < R && (pos < L || pos - L <= trow[r1]) && mrow[j + 1] != -INFINITY;
              e0 = v0 ? e0 : 0.f;
              e1 = v1 ? e1 : 0.f;
            }
            lsum[j] += e0;
            lsum[j + 1] += e1;
            pk[j / 2] = pack_bf16(e0, e1);
          }
          if (n > 0 && !wait_bar(smem_u32(&B->p_free[t]), (n - 1) & 1, abort_flag, p.err, p.wait_limit)) {
            ok = false;
            break;
          }
          // 16-byte chunk cc holds rows 8 cc .. 8 cc + 7: atom cc / (kPAtomRows / 8), chunk
          // cc % (kPAtomRows / 8) of the position's row in that atom
          constexpr int CPA = C::kPAtomRows / 8;   // chunks per atom row
          uint8_t* ptile = smem + C::kPOff + t * C::kPTile + lrow * (C::kPAtomRows * 2);
#pragma unroll
          for (int i = 0; i < NH / 8; ++i) {
            const int cc = sg * (NH / 8) + i;
            *reinterpret_cast<uint4*>(ptile + (cc / CPA) * C::kPAtomBytes + (((cc % CPA) ^ swz_row) << 4)) =
                make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
      if (!ok) break;
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&B->s_empty[n & 1]));
        mbar_arrive(smem_u32(&B->p_full));
      }
      // the previous chunk's output leaves tensor memory (its PV has finished by now or
      // soon: this pass already waited for each of its tiles)
      if (n > 0 && !epilogue(n - 1, xprev)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int j = 0; j < NH; ++j) {
        float sacc = lsum[j];
#pragma unroll
        for (int o = 16; o; o >>= 1) sacc += __shfl_xor_sync(kFull, sacc, o);
        if (lane == j) redL[(sg * 4 + sw4) * NH + j] = sacc;
      }
      if (!wg_sync()) {
        ok = false;
        break;
      }
      if (gt < NH) {
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) l += redL[(sg * 4 + w) * NH + gt];
        cl[(n & 1) * NP + c0 + gt] = l;
      }
      // (cl / redL reuse is ordered by the barriers of the next chunk)
      xprev = x;
    }
    if (ok && n > 0 && !aborted(abort_flag)) {
      if (wg_sync()) epilogue(n - 1, xprev);   // cl of the last chunk complete
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  // the last CTA out returns the counters to zero for the next launch
  if (tid == 0) __threadfence();   // this CTA's claims are performed before its exit count
  if (tid == 0 && atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
    p.sched[0] = 0;
    p.sched[1] = 0;
  }
}

}  // namespace tc

int verify_tc_npad(int R) { return R <= 16 ? 16 : (R <= 32 ? 32 : (R <= 48 ? 48 : (R <= 64 ? 64 : 0))); }

template <int NP>
static int launch_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tk8, const CUtensorMap& tv8, const VerifyParams& p,
                     int batch, int num_sms, cudaStream_t stream) {
  using C = tc::Cfg<NP>;
  static std::atomic<uint64_t> attr_done{0};
  if (cuda_status(ensure_smem_attr(tc::verify_tc_kernel<NP>, C::kSmem, attr_done), "cudaFuncSetAttribute") !=
      S3R_OK)
    return S3R_ERR_CUDA;
  launch_pdl(tc::verify_tc_kernel<NP>, num_sms, tc::kThreads, C::kSmem, stream, tq, tk, tv, tk8, tv8, p,
                                                                        batch);
  return cuda_status(cudaGetLastError(), __func__);
}

bool verify_tc_supported(int D, int R, int /*batch*/) {
  return D == tc::kD && verify_tc_npad(R) != 0;
}

int verify_tc_chunk(int R) {
  const int np = verify_tc_npad(R);
  return np == 16 ? tc::Cfg<16>::kChunk
                   : (np == 32 ? tc::Cfg<32>::kChunk : (np == 48 ? tc::Cfg<48>::kChunk : tc::Cfg<64>::kChunk));
}

// Row pitch of the chunk records: the padded rows for 16 / 32 (as the merge has always read
// them), the real rows (rounded to 4 for 16-byte loads) for 48 and 64, where padding would
// add up to a third to the records' traffic.
int verify_tc_rec_rows(int R) {
  const int np = verify_tc_npad(R);
  return np >= 48 ? (R + 3) / 4 * 4 : np;
}

int launch_verify_tc(const CUtensorMap& qm, const CUtensorMap& k1, const CUtensorMap& v1,
                     const CUtensorMap& k8, const CUtensorMap& v8, const VerifyParams& p,
                     int batch, int num_sms, cudaStream_t stream, int* launches) {
  const int np = verify_tc_npad(p.R);
  *launches = 0;
  if (np != 16 && np != 32 && np != 48 && np != 64) return S3R_ERR_UNSUPPORTED;
  // the per-launch request tables hold kMaxBatch requests; a larger batch is several
  // launches over consecutive slices of it (each chunk record still lands in its slot)
  for (int b0 = 0; b0 < batch; b0 += tc::kMaxBatch) {
    VerifyParams q = p;
    q.req_off = p.req_off + b0;
    const int nb = batch - b0 < tc::kMaxBatch ? batch - b0 : tc::kMaxBatch;
    const int st = np == 16   ? launch_tc<16>(qm, k1, v1, k8, v8, q, nb, num_sms, stream)
                   : np == 32 ? launch_tc<32>(qm, k1, v1, k8, v8, q, nb, num_sms, stream)
                   : np == 48 ? launch_tc<48>(qm, k1, v1, k8, v8, q, nb, num_sms, stream)
                              : launch_tc<64>(qm, k1, v1, k8, v8, q, nb, num_sms, stream);
    if (st != S3R_OK) return st;
    ++*launches;
  }
  return S3R_OK;
}

}  // namespace s3r
