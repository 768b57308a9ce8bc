// Sparse self-draft attention.
//
// What it computes ([News] Interpretation; [Explainer] "How is this different": the draft
// reads a sparse subset of the same KV cache with the same weights): draft step i of
// request r (token at position L+i) writes that token's K/V into its page and lets the G
// query rows of each KV head attend A_i = S ∪ {L, .., L+i}, S the selected positions.
//
// Organisation: a persistent grid (one CTA per SM) over the launch's (request, KV head)
// pairs laid end to end, each pair's A_i positions in order (the selected positions, then
// the block positions). Every CTA computes the pairs' lengths and their prefix sums and
// takes one equal share of the concatenated positions, so every SM gathers the same number
// of rows whatever the lengths; a pair that straddles shares is split into segments (at
// most kSegMax: the share is never below a third of the longest pair), each ending in a
// chunk record, and the CTA that finishes a pair's last segment merges its records.
// Warp roles:
//   warp 0      index warp: per segment it stages the G query rows and the segment's
//               description in a segment slot (and, in the pair's first segment, writes this
//               step's token into its page); per 64-position tile it resolves every
//               position to a pool row (selected index -> page table -> row), kBatchTiles
//               tiles at a time with all their loads in flight, into a ring of row-id slots
//               running up to kOffR tiles ahead of the gather.
//   warps 1-2   gather warps: per tile they copy the 64 K and V rows (256 B each at d = 128)
//               with 16-byte cp.async, 16 lanes per row, into a kNst-stage ring laid out like
//               the verify's TMA tiles (128-byte swizzle); completion is counted on the
//               stage's mbarrier by the copies themselves (cp.async.mbarrier.arrive), so no
//               thread waits on its own loads.
//   warps 3-6   attention warps: the same tensor-core step as the verify (S^T = K Q^T and
//               O^T += V^T P^T by mma.sync, online softmax in log2 units), 16 positions of a
//               tile each; at a segment's end they merge their four states into a record
//               (or straight into the output when the pair has one segment).
// Every wait is on an mbarrier and bounded; an expired wait sets S3R_ERR_TIMEOUT, raises the
// CTA's abort flag, and every role winds down (the gather warps wait for their own copies
// before they exit).
#include "attention.cuh"
#include "kernels.h"

namespace s3r {
namespace dr {

constexpr int kNst = 4;            // K/V ring stages of 64 rows
constexpr int kOffR = 16;          // tile slots of resolved pool rows
constexpr int kSegR = 8;           // segment slots (query rows + description)
constexpr int kBatchTiles = 4;     // tiles the index warp resolves with one set of loads
constexpr int kMaxPairs = 4096;    // (request, KV head) pairs per launch (prefix in shared memory)
constexpr int kGatherWarps = 2;
constexpr int kAttnWarps = 4;
constexpr int kThreads = 32 * (1 + kGatherWarps + kAttnWarps);
constexpr int kRW = 8;             // query rows per record (G <= 8)
constexpr int kAttn0 = 32 * (1 + kGatherWarps);   // first thread of the attention warps

struct TileMeta {
  int nvalid;          // positions of the tile that belong to the segment (<= 64)
  int flags;           // 1: first tile of its segment, 2: last; segment slot << 8
  long long new_off;   // element offset of this pair's new token in k_new / v_new
};
struct SegInfo {
  int r, kvh, pair, j, nseg, pad[3];
};
struct Bars {
  uint64_t full[kNst], empty[kNst];
  uint64_t off_full[kOffR], off_empty[kOffR];
  uint64_t seg_full[kSegR], seg_empty[kSegR];
  uint64_t grp;        // barrier of the attention warps
  int abort_flag;
  int last_flag;
  int amax;
  int pad;
};

template <int D>
struct Lay {
  static constexpr int kStage = 2 * kTile * D * 2;                 // K tile + V tile
  static constexpr int kQBytes = kRW * D * 2;                      // G (<= 8) query rows
  static constexpr int kQOff = kNst * kStage;
  static constexpr int kRedOff = kQOff + kSegR * kQBytes;          // redO [4][8][D+4], redM, redL [4][8]
  static constexpr int kRedBytes = (kAttnWarps * kRW * (D + 4) + 2 * kAttnWarps * kRW) * 4;
  static constexpr int kOffsOff = kRedOff + kRedBytes;             // int32 [kOffR][64]
  static constexpr int kMetaOff = kOffsOff + kOffR * kTile * 4;    // TileMeta [kOffR]
  static constexpr int kSMetaOff = kMetaOff + kOffR * 16;          // TileMeta [kNst]
  static constexpr int kSegOff = kSMetaOff + kNst * 16;            // SegInfo [kSegR]
  static constexpr int kWtsOff = kSegOff + kSegR * 32;             // combine weights
  static constexpr int kWtsFloats = (2 + kSegMax) * kRW;
  static constexpr int kPrefOff = kWtsOff + kWtsFloats * 4;        // int32 [kMaxPairs + 1]
  static constexpr int kScanOff = kPrefOff + (kMaxPairs + 1) * 4;  // int32 [kThreads / 32]
  static constexpr int kBarOff = (kScanOff + 64 + 63) / 64 * 64;
  static constexpr int kSmem = kBarOff + (int)sizeof(Bars) + 1024;  // + alignment slack
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static_assert(kQOff % 1024 == 0 && kRedOff % 16 == 0 && kMetaOff % 16 == 0 && kBarOff % 64 == 0,
                "alignment of the swizzled ring, the query rows and the barriers");
};

__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// The CTA's share of the concatenated positions and its walk over the pairs it touches.
struct Walk {
  const int* pref;
  int npairs, lo, hi;
  int cur;               // next pair to look at
  // The next non-empty segment (pair, its positions [a0, a1) inside this share); false when
  // the share is done. Pairs of length 0 (inputs out of range) are skipped.
  __device__ bool next(int& pair, int& a0, int& a1) {
    while (cur < npairs && (pref[cur + 1] <= lo || pref[cur + 1] == pref[cur])) ++cur;
    if (cur >= npairs || pref[cur] >= hi) return false;
    pair = cur;
    a0 = max(lo, pref[cur]) - pref[cur];
    a1 = min(hi, pref[cur + 1]) - pref[cur];
    ++cur;
    return true;
  }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1) draft_kernel(const DraftParams p, int batch) {
  pdl_wait();
  using Y = Lay<D>;
  constexpr int CPR = D / 8;   // 16-byte chunks per row
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                             ~uintptr_t(1023));
  int* pref = reinterpret_cast<int*>(smem + Y::kPrefOff);
  int* scan = reinterpret_cast<int*>(smem + Y::kScanOff);
  int* offs = reinterpret_cast<int*>(smem + Y::kOffsOff);
  TileMeta* meta = reinterpret_cast<TileMeta*>(smem + Y::kMetaOff);
  TileMeta* smeta = reinterpret_cast<TileMeta*>(smem + Y::kSMetaOff);
  SegInfo* seg = reinterpret_cast<SegInfo*>(smem + Y::kSegOff);
  Bars* B = reinterpret_cast<Bars*>(smem + Y::kBarOff);
  volatile int* abort_flag = &B->abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hkv = p.Hkv, G = p.G;
  const int npairs = batch * Hkv;

  // ---- pair lengths A = n + i + 1 (0 for a pair whose inputs are out of range), their
  // inclusive prefix sums in pref[1..npairs] and the longest A
  if (tid == 0) B->amax = 0;
  __syncthreads();
  const int per = (npairs + kThreads - 1) / kThreads;
  const int q0 = tid * per, q1 = min(npairs, q0 + per);
  int local = 0, amax = 0;
  for (int q = q0; q < q1; ++q) {
    const int b = q / Hkv, h = q - b * Hkv;
    const int r = p.req_ids ? p.req_ids[p.req_off + b] : p.req_off + b;
    int A = 0;
    if (r >= 0 && r < p.num_requests) {
      const int L = p.seq_lens[r], i = p.draft_step[r];
      const int n = p.sel_count[(size_t)r * Hkv + h];
      if (L >= 0 && i >= 0 && i < S3R_MAX_K && L + i < p.cap && n >= 0 && n <= p.sel_stride)
        A = n + i + 1;
    }
    if (A == 0 && blockIdx.x == 0) set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
    pref[q + 1] = A;
    local += A;
    amax = max(amax, A);
  }
  // block scan of the threads' sums (threads own consecutive pairs)
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scan[warp] = incl;
  if (amax) atomicMax(&B->amax, amax);
  __syncthreads();
  int before = 0, total = 0;
  for (int w = 0; w < kThreads / 32; ++w) {
    if (w < warp) before += scan[w];
    total += scan[w];
  }
  int run = before + incl - local;
  for (int q = q0; q < q1; ++q) {
    run += pref[q + 1];
    pref[q + 1] = run;
  }
  if (tid == 0) {
    pref[0] = 0;
    for (int s = 0; s < kNst; ++s) {
      mbar_init(smem_u32(&B->full[s]), 32 * kGatherWarps + 1);
      mbar_init(smem_u32(&B->empty[s]), kAttnWarps);
    }
    for (int s = 0; s < kOffR; ++s) {
      mbar_init(smem_u32(&B->off_full[s]), 1);
      mbar_init(smem_u32(&B->off_empty[s]), kGatherWarps);
    }
    for (int s = 0; s < kSegR; ++s) {
      mbar_init(smem_u32(&B->seg_full[s]), 1);
      mbar_init(smem_u32(&B->seg_empty[s]), 1);
    }
    mbar_init(smem_u32(&B->grp), kAttnWarps);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // ---- this CTA's share [lo, hi) of the P positions
  const int P = total;
  const int A_max = B->amax;
  int share = (P + (int)gridDim.x - 1) / (int)gridDim.x;
  share = max(share, (A_max + kSegMax - 2) / (kSegMax - 1));   // at most kSegMax segments a pair
  share = max(share, kTile);
  const int lo = (int)blockIdx.x * share;
  const int hi = min(P, lo + share);
  if (lo >= hi) return;
  // the pair holding position lo: the last p with pref[p] <= lo
  int p0;
  {
    int a = 0, b = npairs;   // pref[a] <= lo < pref[b]
    while (b - a > 1) {
      const int m = (a + b) >> 1;
      if (pref[m] <= lo) a = m;
      else b = m;
    }
    p0 = a;
  }
  // tiles of this CTA (every role walks the same segments)
  int ntiles = 0;
  {
    Walk w{pref, npairs, lo, hi, p0};
    int pr, a0, a1;
    while (w.next(pr, a0, a1)) ntiles += (a1 - a0 + kTile - 1) / kTile;
  }
  const uint32_t sbase = smem_u32(smem);
  const int wl = p.wait_limit;

  if (warp == 0) {
    // ================================================================ index warp ====
    Walk w{pref, npairs, lo, hi, p0};
    int pr, a0, a1, t = 0, segk = 0;
    bool ok = true;
    while (ok && w.next(pr, a0, a1)) {
      const int b = pr / Hkv, h = pr - b * Hkv;
      const int r = p.req_ids ? p.req_ids[p.req_off + b] : p.req_off + b;
      const int L = p.seq_lens[r], i = p.draft_step[r];
      const int n = p.sel_count[(size_t)r * Hkv + h];
      const int* ptab = p.page_table + (size_t)r * p.max_pages;
      const int* sel = p.sel_idx + ((size_t)r * Hkv + h) * p.sel_stride;
      const size_t new_off = (size_t)r * p.kv_stride + (size_t)h * D;
      const int ss = segk % kSegR;
      if (segk >= kSegR &&
          !wait_bar(smem_u32(&B->seg_empty[ss]), (uint32_t)((segk / kSegR) - 1) & 1u, abort_flag, p.err, wl)) {
        ok = false;
        break;
      }
      // query rows (G of them; rows G..7 zero) and the segment's description
      __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem + Y::kQOff + ss * Y::kQBytes);
      const __nv_bfloat16* qg = p.q + (size_t)r * p.q_stride + (size_t)h * G * D;
      for (int v = lane; v < kRW * CPR; v += 32) {
        const int row = v / CPR, ch = v - row * CPR;
        uint4 x = make_uint4(0, 0, 0, 0);
        if (row < G) x = *reinterpret_cast<const uint4*>(qg + (size_t)row * D + ch * 8);
        *reinterpret_cast<uint4*>(qs + row * D + ch * 8) = x;
      }
      const int cfirst = pref[pr] / share, clast = (pref[pr + 1] - 1) / share;
      if (lane == 0) {
        seg[ss].r = r;
        seg[ss].kvh = h;
        seg[ss].pair = pr;
        seg[ss].j = (int)blockIdx.x - cfirst;
        seg[ss].nseg = clast - cfirst + 1;
      }
      // this step's token enters the cache at position L+i (once per pair; other segments
      // read it from k_new / v_new)
      if (a0 == 0 && lane < CPR) {
        const int pos = L + i;
        const int page = ptab[pos >> 4];
        if (page < 0 || page >= p.num_pages) {
          set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
        } else {
          const size_t dst = (((size_t)page * Hkv + h) * kPage + (pos & 15)) * D + lane * 8;
          *reinterpret_cast<uint4*>(p.k_pool + dst) = *reinterpret_cast<const uint4*>(p.k_new + new_off + lane * 8);
          *reinterpret_cast<uint4*>(p.v_pool + dst) = *reinterpret_cast<const uint4*>(p.v_new + new_off + lane * 8);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&B->seg_full[ss]));
      ++segk;

      // pool rows of the segment's tiles, kBatchTiles tiles per round of loads
      const int ntl = (a1 - a0 + kTile - 1) / kTile;
      for (int tb = 0; tb < ntl && ok; tb += kBatchTiles) {
        const int nb = min(kBatchTiles, ntl - tb);
        for (int u = 0; u < nb; ++u) {
          const int tt = t + u;
          if (tt >= kOffR && !wait_bar(smem_u32(&B->off_empty[tt % kOffR]),
                                       (uint32_t)((tt / kOffR) - 1) & 1u, abort_flag, p.err, wl)) {
            ok = false;
            break;
          }
        }
        if (!ok) break;
        int pos[2 * kBatchTiles], pg[2 * kBatchTiles];
#pragma unroll
        for (int q = 0; q < 2 * kBatchTiles; ++q) {
          const int a = a0 + (tb + (q >> 1)) * kTile + lane + 32 * (q & 1);
          pos[q] = (q >> 1) < nb && a < a1 ? (a < n ? sel[a] : L + (a - n)) : -1;
        }
#pragma unroll
        for (int q = 0; q < 2 * kBatchTiles; ++q)
          pg[q] = (pos[q] >= 0 && pos[q] < L + i) ? ptab[pos[q] >> 4] : -1;   // committed positions
#pragma unroll
        for (int q = 0; q < 2 * kBatchTiles; ++q) {
          const int u = q >> 1;
          if (u >= nb) continue;
          const int a = a0 + (tb + u) * kTile + lane + 32 * (q & 1);
          int row = -1;   // -1: zero row (padding, or a bad index / page, flagged)
          if (a < a1) {
            if (a < n && (pos[q] < 0 || pos[q] >= L)) {
              set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
            } else if (pos[q] == L + i) {
              row = -2;   // this step's token, read from k_new / v_new
            } else if (pg[q] < 0 || pg[q] >= p.num_pages) {
              set_error(p.err, S3R_ERR_DEVICE_BOUNDS);
            } else {
              row = (pg[q] * Hkv + h) * kPage + (pos[q] & 15);
            }
          }
          offs[((t + u) % kOffR) * kTile + lane + 32 * (q & 1)] = row;
        }
        if (lane < nb) {
          const int u = lane, tl = tb + u;
          TileMeta m;
          m.nvalid = min(kTile, a1 - (a0 + tl * kTile));
          m.flags = (tl == 0 ? 1 : 0) | (tl == ntl - 1 ? 2 : 0) | (ss << 8);
          m.new_off = (long long)new_off;
          meta[(t + u) % kOffR] = m;
        }
        __syncwarp();
        if (lane < nb) mbar_arrive(smem_u32(&B->off_full[(t + lane) % kOffR]));
        t += nb;
      }
    }
  } else if (warp <= kGatherWarps) {
    // ============================================================== gather warps ====
    const int ft = tid - 32;   // 0 .. 63
    for (int t = 0; t < ntiles; ++t) {
      const int ts = t % kOffR, s = t % kNst;
      if (!wait_bar(smem_u32(&B->off_full[ts]), (uint32_t)(t / kOffR) & 1u, abort_flag, p.err, wl)) break;
      if (t >= kNst && !wait_bar(smem_u32(&B->empty[s]), (uint32_t)((t / kNst) - 1) & 1u, abort_flag, p.err, wl))
        break;
      const TileMeta m = meta[ts];
      const uint32_t kdst = sbase + s * Y::kStage, vdst = kdst + kTile * D * 2;
      const int* rows = offs + ts * kTile;
      // 16 lanes per 256-byte row (d = 128): each warp instruction covers whole rows
#pragma unroll 4
      for (int mm = 0; mm < CPR; ++mm) {
        const int idx = ft + 32 * kGatherWarps * mm;
        const int row = idx / CPR, ch = idx - row * CPR;
        const int rid = rows[row];
        const __nv_bfloat16 *ks, *vs;
        int bytes = 16;
        if (rid >= 0) {
          ks = p.k_pool + (size_t)rid * D + ch * 8;
          vs = p.v_pool + (size_t)rid * D + ch * 8;
        } else if (rid == -2) {
          ks = p.k_new + m.new_off + ch * 8;
          vs = p.v_new + m.new_off + ch * 8;
        } else {
          ks = p.k_new + m.new_off;   // any valid address; nothing is read, zeros land
          vs = p.v_new + m.new_off;
          bytes = 0;
        }
        cp_async16(kdst + swz(row, ch), ks, bytes);
        cp_async16(vdst + swz(row, ch), vs, bytes);
      }
      cp_async_arrive_noinc(smem_u32(&B->full[s]));   // counts once this thread's copies land
      if (ft == 0) {
        smeta[s] = m;
        mbar_arrive(smem_u32(&B->full[s]));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&B->off_empty[ts]));   // the row ids have been read
    }
    cp_async_wait_all();   // nothing lands in shared memory after this warp exits
  } else {
    // =========================================================== attention warps ====
    const int cw = warp - 1 - kGatherWarps;   // 0..3: positions 16 cw .. 16 cw + 15 of a tile
    const int at = tid - kAttn0;              // 0..127
    float* redO = reinterpret_cast<float*>(smem + Y::kRedOff);
    float* redM = redO + kAttnWarps * kRW * (D + 4);
    float* redL = redM + kAttnWarps * kRW;
    float* wts = reinterpret_cast<float*>(smem + Y::kWtsOff);
    uint32_t grp_phase = 0;
    auto grp_sync = [&]() -> bool {   // the four attention warps (bounded, on an mbarrier)
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&B->grp));
      const bool r = wait_bar(smem_u32(&B->grp), grp_phase, abort_flag, p.err, wl);
      grp_phase ^= 1u;
      return r;
    };
    WarpAttn<D, 1> wa;
    int segk = 0;
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kNst;
      if (!wait_bar(smem_u32(&B->full[s]), (uint32_t)(t / kNst) & 1u, abort_flag, p.err, wl)) break;
      const TileMeta m = smeta[s];
      const int ss = m.flags >> 8;
      if (m.flags & 1) {
        if (!wait_bar(smem_u32(&B->seg_full[ss]), (uint32_t)(segk / kSegR) & 1u, abort_flag, p.err, wl)) break;
        const __nv_bfloat16* qs = reinterpret_cast<const __nv_bfloat16*>(smem + Y::kQOff + ss * Y::kQBytes);
        wa.init();
        wa.load_q(0, lane, [&](int rr) -> const __nv_bfloat16* { return rr < G ? qs + rr * D : nullptr; });
      }
      const uint32_t kb = sbase + s * Y::kStage, vb = kb + kTile * D * 2;
      const int row0 = cw * 16, nv = m.nvalid;
      if (row0 < nv) {
        auto vis = [&](int tr, int, int) -> bool { return tr < nv; };
        auto nocap = [](int, int, float, float) {};
        if (nv >= kTile)
          wa.template step<false>(kb, vb, row0, lane, p.scale, vis, nocap);
        else
          wa.template step<true>(kb, vb, row0, lane, p.scale, vis, nocap);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&B->empty[s]));
      if (!(m.flags & 2)) continue;

      // ---- end of a segment: merge the four warps' states
      const SegInfo si = seg[ss];
      wa.finish_sums();
      wa.store_shared(redO, redM, redL, cw, lane);
      if (!grp_sync()) break;
      const int r = si.r, h = si.kvh;
      auto out_row = [&](int row) { return p.out + ((size_t)r * p.Hq + h * G + row) * D; };
      auto lse_row = [&](int row) -> float* { return p.lse ? p.lse + (size_t)r * p.Hq + h * G + row : nullptr; };
      if (si.nseg == 1) {
        // the whole pair is here: normalise straight into the output
        for (int idx = at; idx < G * (D / 2); idx += 32 * kAttnWarps) {
          const int row = idx / (D / 2), d2 = (idx - row * (D / 2)) * 2;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, redM[w * kRW + row]);
          float a0 = 0.f, a1 = 0.f, ls = 0.f;
#pragma unroll
          for (int w = 0; w < kAttnWarps; ++w) {
            const float mw = redM[w * kRW + row];
            const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
            const float* o = redO + ((size_t)w * kRW + row) * (D + 4) + d2;
            a0 += f * o[0];
            a1 += f * o[1];
            ls += f * redL[w * kRW + row];
          }
          const float il = 1.f / ls;
          *reinterpret_cast<__nv_bfloat162*>(out_row(row) + d2) = __floats2bfloat162_rn(a0 * il, a1 * il);
          float* lp = lse_row(row);
          if (d2 == 0 && lp) *lp = (M + log2f(ls)) * kLn2;
        }
      } else {
        const size_t rec_floats = (size_t)kRW * (D + 2);
        float* recs = p.part + ((size_t)r * Hkv + h) * kSegMax * rec_floats;
        merge_slices_to_record<D, kRW>(redO, redM, redL, 1, recs + (size_t)si.j * rec_floats, kRW, at,
                                       32 * kAttnWarps);
        __threadfence();
        if (!grp_sync()) break;
        if (at == 0) {
          int* ticket = p.tickets + (size_t)r * Hkv + h;
          const int prev = atomicAdd(ticket, 1);
          B->last_flag = prev == si.nseg - 1;
          if (B->last_flag) *ticket = 0;
        }
        if (!grp_sync()) break;
        if (B->last_flag) {
          __threadfence();
          bool sync_ok = true;
          combine_records_sync<D>(recs, rec_floats, si.nseg, G, kRW, wts, Y::kWtsFloats, out_row, lse_row, at,
                                  32 * kAttnWarps, [&] { sync_ok = grp_sync() && sync_ok; });
          if (!sync_ok) break;
        }
      }
      // the reduction scratch and the segment slot are free again
      if (!grp_sync()) break;
      if (at == 0) mbar_arrive(smem_u32(&B->seg_empty[ss]));
      ++segk;
    }
  }
}

}  // namespace dr

template <int D>
static int launch_draft_d(const DraftParams& p, int batch, int num_sms, cudaStream_t stream, int* launches) {
  using Y = dr::Lay<D>;
  static std::atomic<uint64_t> attr_done{0};
  if (cuda_status(ensure_smem_attr(dr::draft_kernel<D>, Y::kSmem, attr_done), "cudaFuncSetAttribute") != S3R_OK)
    return S3R_ERR_CUDA;
  // the pair prefix lives in shared memory: larger batches are several launches over
  // consecutive request slices (records and tickets are per request, so slices are independent)
  const int per_launch = dr::kMaxPairs / p.Hkv;
  for (int b0 = 0; b0 < batch; b0 += per_launch) {
    DraftParams q = p;
    q.req_off = p.req_off + b0;
    const int nb = batch - b0 < per_launch ? batch - b0 : per_launch;
    launch_pdl(dr::draft_kernel<D>, num_sms, dr::kThreads, Y::kSmem, stream, q, nb);
    const int st = cuda_status(cudaGetLastError(), __func__);
    if (st != S3R_OK) return st;
    ++*launches;
  }
  return S3R_OK;
}

int launch_draft(const DraftParams& p, int D, int batch, int num_sms, cudaStream_t stream, int* launches) {
  *launches = 0;
  if (D == 128) return launch_draft_d<128>(p, batch, num_sms, stream, launches);
  if (D == 64) return launch_draft_d<64>(p, batch, num_sms, stream, launches);
  return S3R_ERR_UNSUPPORTED;
}

size_t draft_partial_bytes(int num_requests, int Hkv, int /*sel_stride*/, int D) {
  return align_up((size_t)num_requests * Hkv * kSegMax * dr::kRW * (D + 2) * 4, 256);
}

}  // namespace s3r
