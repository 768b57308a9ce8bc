// Device helpers shared by the S3R kernels: PTX wrappers for sm_100a (ldmatrix, mma.sync,
// movmatrix, cp.async, mbarrier, TMA tiled and untiled bulk loads, programmatic dependent
// launch), warp reductions, Philox4x32-10 and the workspace layout.
#pragma once

#include <atomic>
#include <utility>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/s3r.h"

namespace s3r {

constexpr int kPage = 16;
constexpr int kTile = 64;                 // KV positions per pipeline stage
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kWaitLimit = 1 << 24;       // bounded spin on an mbarrier phase (default)

// ---------------------------------------------------------------- workspace layout ----
// [0, 256)      error word (int32 bitmask of 1 << s3r_status) at 0; at 64 the dense verify's
//               work counter and exit counter (zero between calls); the rest reserved
// [256, T)      tickets: int32 [num_requests][kMaxKvHeads] (zero between calls); the same
//               region for every call, whatever its head count
// [T, ...)      per-call partials, overwritten by each call
constexpr size_t kWsHeader = 256;
constexpr size_t kWsSchedOff = 64;
constexpr int kMaxKvHeads = 64;
__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline size_t ws_tickets_bytes(int num_requests) {
  return align_up((size_t)num_requests * kMaxKvHeads * 4, 256);
}

__device__ __forceinline__ void set_error(int* err, int code) { atomicOr(err, 1 << code); }

// ------------------------------------------------------------------------ PTX ----------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose an 8x8 b16 matrix held in the ldmatrix fragment layout across the warp.
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// Two floats -> bf16x2 (round to nearest even); `lo` lands in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// cp.async 16 bytes global -> shared; src_bytes == 0 fills zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of a phase.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and the caller records S3R_ERR_TIMEOUT) if the phase
// did not complete within kWaitLimit polls.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (int i = 0; i < kWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Warp-uniform bounded wait on an mbarrier phase (every lane observes the phase itself).
// Gives up when another role raised the abort flag, or after `limit` polls (then raises
// it, with S3R_ERR_TIMEOUT in the error word). For waits on another role's progress; a
// wait for this thread's own copies or tensor-core work in flight uses mbar_wait, which
// no abort cuts short.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int* err, int limit = kWaitLimit) {
  for (int i = 0; i < limit; ++i) {
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
// Programmatic dependent launch: every kernel of the library is launched with the
// programmatic-stream-serialization attribute and waits here, before its first access to
// global memory, until the preceding kernel of the stream has completed and its writes are
// visible. Stream order is therefore unchanged; what overlaps is the next launch's set-up
// (grid launch, CTA placement) with the previous kernel's tail. Without a preceding
// programmatic launch the wait returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline void launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  (void)cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);   // errors: cudaGetLastError
}

// Raise `kern`'s dynamic shared-memory limit to `bytes` on the current device, once per
// device: the attribute belongs to the device, so a process that drives several GPUs sets
// it on each. `done` is the caller's record (bit d: device d done; devices >= 64 set it on
// every call). Returns the CUDA error of the attribute call.
template <typename... KArgs>
inline cudaError_t ensure_smem_attr(void (*kern)(KArgs...), int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t)1 << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Untiled bulk copy global -> shared of `bytes` (both addresses 16-byte aligned, bytes a
// multiple of 16), completion counted on `bar` (bytes).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// 2-D TMA tiled load global -> shared, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// 3-D TMA tiled load global -> shared (coordinates innermost first).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// 4-D TMA tiled load global -> shared (coordinates innermost first).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            int z, int w, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
      : "memory");
}

// Byte offset of 16-byte chunk `c` (0 .. d/8-1) of tile row `row` in a stage laid out as
// [d/64 halves][kTile rows][128 B] with the 128-byte swizzle (chunk ^= row % 8), the layout a
// TMA load with CU_TENSOR_MAP_SWIZZLE_128B writes into a 1024-byte aligned buffer.
__device__ __forceinline__ uint32_t swz(int row, int c) {
  return (uint32_t)((c >> 3) * (kTile * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// ------------------------------------------------------------------- reductions -------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Merge two (max, sum of exp(x - max)) pairs; the sum is kept in double.
__device__ __forceinline__ void merge_ms(float& m, double& s, float m2, double s2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) { m = m2; s = s2; return; }
  if (m2 > m) { s = s * exp((double)m - (double)m2) + s2; m = m2; }
  else { s += s2 * exp((double)m2 - (double)m); }
}

// Count this CTA's chunk on the ticket of its (request, KV head); true in the CTA that
// completes the set (which then owns the combine and resets the ticket).
__device__ __forceinline__ bool last_of(int* ticket, int total, int* s_flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(ticket, 1);
    *s_flag = (prev == total - 1);
    if (*s_flag) *ticket = 0;
  }
  __syncthreads();
  const bool last = *s_flag != 0;
  if (last) __threadfence();
  return last;
}

// --------------------------------------------------------------------- Philox ---------
// Philox4x32-10 (Salmon et al., SC'11): 10 rounds, multipliers 0xD2511F53 / 0xCD9E8D57,
// key bumps 0x9E3779B9 / 0xBB67AE85.
__host__ __device__ inline void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
  for (int i = 0; i < 10; ++i) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

// u in [0,1) with 24 random bits, from counter (position, request, stream, 0).
__device__ __forceinline__ double philox_u(uint64_t seed, uint32_t position, uint32_t request,
                                           uint32_t stream) {
  uint32_t c[4] = {position, request, stream, 0u};
  philox4x32_10(c, (uint32_t)seed, (uint32_t)(seed >> 32));
  return (double)(c[0] >> 8) * (1.0 / 16777216.0);
}

}  // namespace s3r
